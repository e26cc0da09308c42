// Main Branch, KV-outer (pnsm.cn explainer sec. 7 "KV-outer sparse attention",
// "query gather", "two-phase combine"; yhxrc.cn sec. 二: loop over KV blocks and
// gather every query that chose the block, so each block is read once;
// yololab.net "KV Outer Gather Q").
//
// A pass over query rows [t0, t1):
//   1. count    : per (sequence, group, block) list, how many (query, slot)
//                 entries chose it (warp-aggregated atomics);
//   2. plan     : exclusive scans -> list offsets, work items of at most
//                 `queries_per_item` queries per list;
//   3. scatter  : list entries (t - t0) * k + slot;
//   4. attend   : one work item = one KV block (TMA, loaded once) and up to
//                 queries_per_item gathered queries; per 128-row tile
//                 (128 / Hg queries x Hg heads) S = Q K^T and O = P V run on
//                 tcgen05 with fp32 accumulators in TMEM; each (query, group,
//                 block) writes its normalised output (f16) and log-sum-exp;
//   5. combine  : per (query, head) log-sum-exp merge of its partials.
#include "msa_common.cuh"

namespace msa {
namespace {

// ------------------------------------------------------------- helpers ---

__device__ __forceinline__ int find_seq(const int32_t* __restrict__ cu, int batch, int64_t row) {
  int lo = 0, hi = batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu[mid] <= row) lo = mid; else hi = mid;
  }
  return lo;
}

__global__ void block_offsets_kernel(const int32_t* __restrict__ cu_k, int batch, int32_t* __restrict__ blk_off) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    int acc = 0;
    for (int b = 0; b < batch; ++b) {
      blk_off[b] = acc;
      acc += (cu_k[b + 1] - cu_k[b] + kBk - 1) / kBk;
    }
    blk_off[batch] = acc;
  }
}

// Validates an entry and returns its list id, or -1 (slot empty or invalid).
__device__ __forceinline__ int entry_list(int blk, int64_t t, int g, int G, int batch, const int32_t* cu_q,
                                          const int32_t* cu_k, const int32_t* blk_off, DevError* err, int* seq_out) {
  if (blk < 0) return -1;
  const int b = find_seq(cu_q, batch, t);
  const int Tb = cu_q[b + 1] - cu_q[b];
  const int Sb = cu_k[b + 1] - cu_k[b];
  const int64_t pos = (int64_t)Sb - Tb + (t - cu_q[b]);
  if (Tb > Sb || blk > pos / kBk) {
    report_error(err, MSA_ERR_DEVICE_CHECK, kSiteInvert, (int)t, blk);
    return -1;
  }
  *seq_out = b;
  return (blk_off[b] + blk) * G + g;
}

// Pass 1 and 3: one thread per (query, group).  scatter == false counts,
// scatter == true claims positions from `cursor` and writes the entries.
template <bool kScatter>
__global__ void count_scatter_kernel(const int32_t* __restrict__ sel, int64_t t0, int64_t t1, int G, int k,
                                     int batch, const int32_t* __restrict__ cu_q, const int32_t* __restrict__ cu_k,
                                     const int32_t* __restrict__ blk_off, int32_t* __restrict__ counter,
                                     uint32_t* __restrict__ entries, DevError* err) {
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t n = (t1 - t0) * G;
  const bool active = gid < n;
  const int64_t t = t0 + (active ? gid / G : 0);
  const int g = active ? (int)(gid % G) : 0;
  const int lane = threadIdx.x & 31;
  for (int s = 0; s < k; ++s) {
    int L = -1, seq = 0;
    if (active) L = entry_list(sel[(t * G + g) * k + s], t, g, G, batch, cu_q, cu_k, blk_off, err, &seq);
    // warp-aggregated atomics: lanes with the same list share one atomic
    const unsigned peers = __match_any_sync(0xffffffffu, L);
    const int leader = __ffs(peers) - 1;
    const int rank = __popc(peers & ((1u << lane) - 1u));
    int base = 0;
    if (L >= 0 && lane == leader) base = atomicAdd(&counter[L], __popc(peers));
    base = __shfl_sync(0xffffffffu, base, leader);
    if (kScatter && L >= 0) entries[base + rank] = (uint32_t)((t - t0) * k + s);
  }
}

// Pass 2: one CTA.  offsets = exclusive scan of counts; items per list =
// ceil(count / C); cursor = offsets (for the scatter); then the items.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* __restrict__ counts, int64_t nlists, int G,
                                                    int batch, const int32_t* __restrict__ blk_off, int C,
                                                    int32_t* __restrict__ offsets, int32_t* __restrict__ cursor,
                                                    int32_t* __restrict__ item_off, int32_t* __restrict__ nitems,
                                                    Item* __restrict__ items, int64_t max_items, DevError* err) {
  __shared__ int32_t warp_a[32], warp_b[32];
  __shared__ int32_t carry_a, carry_b;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  if (tid == 0) { carry_a = 0; carry_b = 0; }
  __syncthreads();
  for (int64_t base = 0; base < nlists; base += 1024) {
    const int64_t L = base + tid;
    const int c = L < nlists ? counts[L] : 0;
    const int ni = (c + C - 1) / C;
    int a = c, b = ni;  // inclusive warp scans
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ya = __shfl_up_sync(0xffffffffu, a, o), yb = __shfl_up_sync(0xffffffffu, b, o);
      if (lane >= o) { a += ya; b += yb; }
    }
    if (lane == 31) { warp_a[wid] = a; warp_b[wid] = b; }
    __syncthreads();
    if (wid == 0) {
      int wa = warp_a[lane], wb = warp_b[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int ya = __shfl_up_sync(0xffffffffu, wa, o), yb = __shfl_up_sync(0xffffffffu, wb, o);
        if (lane >= o) { wa += ya; wb += yb; }
      }
      warp_a[lane] = wa;
      warp_b[lane] = wb;
    }
    __syncthreads();
    const int pa = carry_a + (wid ? warp_a[wid - 1] : 0) + a - c;
    const int pb = carry_b + (wid ? warp_b[wid - 1] : 0) + b - ni;
    if (L < nlists) {
      offsets[L] = pa;
      cursor[L] = pa;
      item_off[L] = pb;
    }
    __syncthreads();
    if (tid == 1023) { carry_a = pa + c; carry_b = pb + ni; }
    __syncthreads();
  }
  if (tid == 0) {
    offsets[nlists] = carry_a;
    item_off[nlists] = carry_b;
    *nitems = carry_b <= max_items ? carry_b : 0;
    if (carry_b > max_items) report_error(err, MSA_ERR_WORKSPACE, kSiteInvert, carry_b, (int)max_items);
  }
  __syncthreads();
  if (item_off[nlists] > max_items) return;
  // items
  for (int64_t L = tid; L < nlists; L += 1024) {
    const int c = counts[L];
    if (c == 0) continue;
    const int gb = (int)(L / G), g = (int)(L % G);
    int lo = 0, hi = batch;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (blk_off[mid] <= gb) lo = mid; else hi = mid;
    }
    const int off = offsets[L];
    int io = item_off[L];
    for (int s = 0; s < c; s += C, ++io) {
      Item it;
      it.seq = lo;
      it.blk = gb - blk_off[lo];
      it.g = g;
      it.start = off + s;
      it.count = min(C, c - s);
      it.pad0 = it.pad1 = it.pad2 = 0;
      items[io] = it;
    }
  }
}

// ------------------------------------------------------------ attention ---
//
// Warp-specialised, persistent (one CTA per SM, 384 threads):
//   warp 0      claims work items (atomic ticket), publishes them in a 4-deep
//               ring and TMA-loads each item's K and V block into one of two
//               shared-memory stages;
//   warp 1      owns TMEM (512 columns = two slots of S/P + O) and issues the
//               MMAs: S(t+1) = Q K^T is issued before O(t) = P V so the
//               tensor core works while tile t's softmax runs;
//   warps 2-3   gather the Q rows of each 128-row tile (cp.async, 16-byte
//               chunks into the 128-byte-swizzled K-major layout), 3 slots;
//   warps 4-7   softmax + epilogue of even tiles (TMEM slot 0),
//   warps 8-11  the same for odd tiles (slot 1): S -> P (bf16, written back
//               into the S columns, the A operand of the PV MMA), then O / l
//               -> f16 partial and the log-sum-exp of each row.

constexpr int kAttnThreads = 384;
constexpr int kItemRing = 4;
constexpr int kQSlots = 3;
constexpr int kItemEmptyCount = 11;   // gather warps 2 + MMA 1 + softmax warps 8

struct __align__(16) RingItem {
  int32_t seq, blk, g, start, count, pad0, pad1, pad2;
};

struct __align__(16) AttnCtl {
  uint64_t item_full[kItemRing], item_empty[kItemRing];
  uint64_t kv_full[2], kv_empty[2];
  uint64_t q_full[kQSlots], q_empty[kQSlots];
  uint64_t s_full[2], p_full[2], o_full[2], o_free[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int32_t abort_flag;
  int32_t pad[2];
  RingItem ring[kItemRing];
};

// Byte offset of 16-byte chunk `col` (along the 2*D-byte row) of row `row` in a
// K-major [128 x D] bf16 tile stored as D/64 column halves of [128 x 128 B]
// with the 128-byte swizzle.
__device__ __forceinline__ uint32_t kmajor_off(int row, int col) {
  return (col >> 3) * (128 * 128) + swz_offset(row, col & 7, 128);
}

struct TileRef {
  int tau;        // tile counter of this CTA
  int item_seq;   // item counter of this CTA
  bool first, last;
};

__global__ void __launch_bounds__(kAttnThreads, 1)
sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __nv_bfloat16* __restrict__ q, const Item* __restrict__ items,
                   const int32_t* __restrict__ nitems_p, int32_t* __restrict__ ticket,
                   const uint32_t* __restrict__ entries, const int32_t* __restrict__ cu_q,
                   const int32_t* __restrict__ cu_k, int H, int G, int d, int k, float scale_log2,
                   int64_t t0, __half* __restrict__ part_acc, float* __restrict__ part_lse, DevError* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const int tile_bytes = 128 * d * 2;         // one [128 x d] bf16 tile
  uint8_t* kv_s = smem;                        // 2 stages x (K, V)
  uint8_t* q_s = kv_s + 4 * tile_bytes;        // kQSlots tiles
  AttnCtl* ctl = reinterpret_cast<AttnCtl*>(q_s + kQSlots * tile_bytes);
  volatile int32_t* abort_flag = &ctl->abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hg = H / G;
  const int qpt = 128 / Hg;                    // queries per 128-row tile
  const int nhalf = d / 64;
  const int nitems = *nitems_p;

  if (tid == 0) {
    for (int i = 0; i < kItemRing; ++i) { mbar_init(&ctl->item_full[i], 1); mbar_init(&ctl->item_empty[i], kItemEmptyCount); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->kv_full[i], 1); mbar_init(&ctl->kv_empty[i], 1);
      mbar_init(&ctl->s_full[i], 1); mbar_init(&ctl->p_full[i], 4);
      mbar_init(&ctl->o_full[i], 1); mbar_init(&ctl->o_free[i], 4);
    }
    for (int i = 0; i < kQSlots; ++i) { mbar_init(&ctl->q_full[i], 2); mbar_init(&ctl->q_empty[i], 1); }
    mbar_init(&ctl->mma_done, 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  // Reads the next ring item (every consumer warp calls this in the same order).
  // whole_warp: all 32 lanes call it (else only lane 0 of the warp does).
  auto take_item = [&](int n, RingItem& out, bool whole_warp) -> bool {
    const int slot = n % kItemRing;
    if (!mbar_wait(&ctl->item_full[slot], (n / kItemRing) & 1)) {
      report_error(err, MSA_ERR_TIMEOUT, kSiteAttnItem, n, warp);
      *abort_flag = 1;
      return false;
    }
    out = ctl->ring[slot];
    if (whole_warp) __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->item_empty[slot]);
    return out.count > 0;
  };

  if (warp == 0) {
    // ------------------------------------------------ scheduler + K/V loads
    if (lane == 0) {
      int n = 0;
      while (true) {
        const int slot = n % kItemRing;
        if (!mbar_wait(&ctl->item_empty[slot], ((n / kItemRing) + 1) & 1)) {
          report_error(err, MSA_ERR_TIMEOUT, kSiteAttnLoad, n, 0);
          *abort_flag = 1;
          break;
        }
        const int it = *abort_flag ? nitems : atomicAdd(ticket, 1);
        RingItem r;
        if (it >= nitems) {
          r.count = 0;
          ctl->ring[slot] = r;
          mbar_arrive(&ctl->item_full[slot]);
          break;
        }
        const Item I = items[it];
        r.seq = I.seq; r.blk = I.blk; r.g = I.g; r.start = I.start; r.count = I.count;
        ctl->ring[slot] = r;
        mbar_arrive(&ctl->item_full[slot]);
        const int st = n & 1;
        if (!mbar_wait(&ctl->kv_empty[st], ((n >> 1) + 1) & 1)) {
          report_error(err, MSA_ERR_TIMEOUT, kSiteAttnLoad, n, 1);
          *abort_flag = 1;
          break;
        }
        uint8_t* ks = kv_s + st * 2 * tile_bytes;
        mbar_arrive_expect_tx(&ctl->kv_full[st], 2 * tile_bytes);
        const int krow = cu_k[I.seq] + I.blk * kBk;
        for (int h = 0; h < nhalf; ++h) {
          tma_load_3d(ks + h * 128 * 128, &tm_k, &ctl->kv_full[st], 64 * h, I.g, krow);
          tma_load_3d(ks + tile_bytes + h * 128 * 128, &tm_v, &ctl->kv_full[st], 64 * h, I.g, krow);
        }
        ++n;
      }
      // no K/V load may still be in flight when the CTA exits
      for (int st = 0; st < 2; ++st) {
        const int issued = n > st ? (n - st + 1) / 2 : 0;
        if (issued > 0) mbar_wait(&ctl->kv_full[st], (issued - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t idesc_o = idesc_bf16_f32(128, d, 0, 1);
      int n = 0, tau = 0;
      RingItem cur;
      int cur_tiles = 0, mt = 0, cur_seq = -1;
      bool have = false, ok = true;
      // next tile in the stream (consumes items as needed)
      auto next_tile = [&](TileRef& tr) -> bool {
        if (!have || mt >= cur_tiles) {
          if (!take_item(n, cur, false)) return false;
          cur_seq = n++;
          cur_tiles = (cur.count + qpt - 1) / qpt;
          mt = 0;
          have = true;
        }
        tr.tau = tau++;
        tr.item_seq = cur_seq;
        tr.first = (mt == 0);
        tr.last = (mt == cur_tiles - 1);
        ++mt;
        return true;
      };
      auto issue_s = [&](const TileRef& tr) -> bool {
        const int qs = tr.tau % kQSlots, s = tr.tau & 1, st = tr.item_seq & 1;
        if (!mbar_wait(&ctl->q_full[qs], (tr.tau / kQSlots) & 1)) return false;
        if (tr.first && !mbar_wait(&ctl->kv_full[st], (tr.item_seq >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t qa = smem_u32(q_s + qs * tile_bytes), ka = smem_u32(kv_s + st * 2 * tile_bytes);
        for (int kk = 0; kk < d / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
          umma_bf16_ss(tmem + s * 256, make_sdesc(qa + off, 16, 1024, kSw128), make_sdesc(ka + off, 16, 1024, kSw128),
                       idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&ctl->s_full[s]);
        umma_commit(&ctl->q_empty[qs]);
        return true;
      };
      auto issue_pv = [&](const TileRef& tr) -> bool {
        const int s = tr.tau & 1, st = tr.item_seq & 1;
        if (!mbar_wait(&ctl->p_full[s], (tr.tau >> 1) & 1)) return false;
        if (!mbar_wait(&ctl->o_free[s], ((tr.tau >> 1) + 1) & 1)) return false;
        tc_fence_after();
        const uint32_t va = smem_u32(kv_s + st * 2 * tile_bytes + tile_bytes);
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16_ts(tmem + s * 256 + 128, tmem + s * 256 + kk * 8,
                       make_sdesc(va + kk * 2048, 128 * 128, 1024, kSw128), idesc_o, kk > 0 ? 1u : 0u);
        umma_commit(&ctl->o_full[s]);
        if (tr.last) umma_commit(&ctl->kv_empty[st]);
        return true;
      };
      TileRef t0r, t1r;
      if (next_tile(t0r)) {
        ok = issue_s(t0r);
        while (ok && !*abort_flag) {
          const bool more = next_tile(t1r);
          if (more && !(ok = issue_s(t1r))) break;
          if (!(ok = issue_pv(t0r))) break;
          if (!more) break;
          t0r = t1r;
        }
      }
      if (!ok) {
        report_error(err, MSA_ERR_TIMEOUT, kSiteAttnMma, tau, n);
        *abort_flag = 1;
      }
      umma_commit(&ctl->mma_done);
      mbar_wait(&ctl->mma_done, 0);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ Q gather
    const int gt = tid - 64;                   // 0..63
    const int cpr = d / 8;                     // 16-byte chunks per row
    int n = 0, tau = 0;
    RingItem I;
    while (!*abort_flag && take_item(n++, I, true)) {
      const int ntiles = (I.count + qpt - 1) / qpt;
      for (int mt = 0; mt < ntiles; ++mt, ++tau) {
        const int qs = tau % kQSlots;
        if (!mbar_wait(&ctl->q_empty[qs], ((tau / kQSlots) + 1) & 1)) {
          report_error(err, MSA_ERR_TIMEOUT, kSiteAttnLoad, tau, 2);
          *abort_flag = 1;
          break;
        }
        const int nq = min(qpt, I.count - mt * qpt);
        uint8_t* dst = q_s + qs * tile_bytes;
        const uint32_t* ent = entries + I.start + mt * qpt;
        for (int c = gt; c < nq * Hg * cpr; c += 64) {
          const int row = c / cpr, col = c - row * cpr;
          const int ql = row / Hg, i = row - ql * Hg;
          const int64_t t = t0 + ent[ql] / k;
          cp_async_16(dst + kmajor_off(row, col), q + ((t * H) + (int64_t)I.g * Hg + i) * d + col * 8);
        }
        cp_async_commit();
        cp_async_wait_all();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->q_full[qs]);
      }
    }
  } else {
    // ------------------------------------------------- softmax + epilogue
    const int wg = (warp - 4) >> 2;           // slot handled by this warpgroup
    const int wq = warp & 3;                  // TMEM lane quarter
    const int r = 32 * wq + lane;             // tile row
    const uint32_t lane_off = static_cast<uint32_t>(32 * wq) << 16;
    const uint32_t s_col = tmem + wg * 256 + lane_off;      // S, then P (first 64 columns)
    const uint32_t o_col = s_col + 128;                     // O
    const int ql = r / Hg, hi = r - ql * Hg;
    int n = 0, tau = 0;
    RingItem I;
    while (!*abort_flag && take_item(n++, I, true)) {
      const int ntiles = (I.count + qpt - 1) / qpt;
      const int Tb = cu_q[I.seq + 1] - cu_q[I.seq];
      const int Sb = cu_k[I.seq + 1] - cu_k[I.seq];
      const int64_t qrow0 = cu_q[I.seq];
      const int64_t blk_first = (int64_t)I.blk * kBk;
      for (int mt = 0; mt < ntiles; ++mt, ++tau) {
        if ((tau & 1) != wg) continue;
        const int nq = min(qpt, I.count - mt * qpt);
        const bool valid = ql < nq;
        uint32_t e = 0;
        int limit = 127;
        if (valid) {
          e = entries[I.start + mt * qpt + ql];
          const int64_t t = t0 + e / k;
          const int64_t lim = (int64_t)Sb - Tb + (t - qrow0) - blk_first;
          limit = lim >= 127 ? 127 : (int)lim;
        }
        if (!mbar_wait(&ctl->s_full[wg], (tau >> 1) & 1)) {
          report_error(err, MSA_ERR_TIMEOUT, kSiteAttnSoftmax, tau, 0);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        uint32_t rr[32];
        float m = -INFINITY;
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
          tmem_ld32(s_col + 32 * c4, rr);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (32 * c4 + j <= limit) m = fmaxf(m, __uint_as_float(rr[j]));
        }
        const float ms = m * scale_log2;
        float l = 0.f;
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
          tmem_ld32(s_col + 32 * c4, rr);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int c0 = 32 * c4 + 2 * j;
            const float p0 = c0 <= limit ? exp2f(fmaf(__uint_as_float(rr[2 * j]), scale_log2, -ms)) : 0.f;
            const float p1 = c0 + 1 <= limit ? exp2f(fmaf(__uint_as_float(rr[2 * j + 1]), scale_log2, -ms)) : 0.f;
            l += p0 + p1;
            pk[j] = pack_bf16x2(p0, p1);
          }
          tmem_st16(s_col + 16 * c4, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->p_full[wg]);
        // ---- epilogue: O / l -> f16 partial, lse
        if (!mbar_wait(&ctl->o_full[wg], (tau >> 1) & 1)) {
          report_error(err, MSA_ERR_TIMEOUT, kSiteAttnSoftmax, tau, 1);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const float inv_l = 1.f / l;
        const int64_t unit = valid ? ((int64_t)(e / k) * G + I.g) * k + (e % k) : 0;
        __half* dst = part_acc + (unit * Hg + hi) * d;
        for (int c4 = 0; c4 < d / 32; ++c4) {
          tmem_ld32(o_col + 32 * c4, rr);
          tmem_ld_wait();
          if (valid) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint4 w;
              w.x = pack_f16x2(__uint_as_float(rr[8 * j + 0]) * inv_l, __uint_as_float(rr[8 * j + 1]) * inv_l);
              w.y = pack_f16x2(__uint_as_float(rr[8 * j + 2]) * inv_l, __uint_as_float(rr[8 * j + 3]) * inv_l);
              w.z = pack_f16x2(__uint_as_float(rr[8 * j + 4]) * inv_l, __uint_as_float(rr[8 * j + 5]) * inv_l);
              w.w = pack_f16x2(__uint_as_float(rr[8 * j + 6]) * inv_l, __uint_as_float(rr[8 * j + 7]) * inv_l);
              *reinterpret_cast<uint4*>(dst + 32 * c4 + 8 * j) = w;
            }
          }
        }
        if (valid) part_lse[unit * Hg + hi] = (ms + __log2f(l)) * 0.69314718055994530942f;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->o_free[wg]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// -------------------------------------------------------------- combine ---

// One group of d/8 threads per (query, head); each thread owns 8 output
// columns.  Slots with sel < 0 carry no partial.
__global__ void combine_kernel(const __half* __restrict__ part_acc, const float* __restrict__ part_lse,
                               const int32_t* __restrict__ sel, __nv_bfloat16* __restrict__ out,
                               float* __restrict__ lse_out, int64_t T, int H, int G, int d, int k) {
  const int tpr = d / 8;                       // threads per (query, head)
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t pair = gid / tpr;
  const int c = (int)(gid % tpr);
  if (pair >= T * H) return;
  const int64_t t = pair / H;
  const int h = (int)(pair % H);
  const int Hg = H / G, g = h / Hg, i = h % Hg;
  const int32_t* srow = sel + (t * G + g) * k;
  const int64_t ubase = (t * G + g) * k;
  float m = -INFINITY;
  for (int s = 0; s < k; ++s)
    if (srow[s] >= 0) m = fmaxf(m, part_lse[(ubase + s) * Hg + i]);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float wsum = 0.f;
  for (int s = 0; s < k; ++s) {
    if (srow[s] < 0) continue;
    const float w = __expf(part_lse[(ubase + s) * Hg + i] - m);
    wsum += w;
    const uint4 raw = *reinterpret_cast<const uint4*>(part_acc + ((ubase + s) * Hg + i) * d + 8 * c);
    const __half2* hp = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = __half22float2(hp[j]);
      acc[2 * j] += w * f.x;
      acc[2 * j + 1] += w * f.y;
    }
  }
  const float inv = 1.f / wsum;
  uint4 o;
  o.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  o.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
  o.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
  o.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
  *reinterpret_cast<uint4*>(out + (t * H + h) * d + 8 * c) = o;
  if (lse_out != nullptr && c == 0) lse_out[t * H + h] = m + __logf(wsum);
}

}  // namespace

// -------------------------------------------------------------- launchers ---

int launch_sparse_attn_pass(const AttnArgs& a, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t nrows = a.t1 - a.t0;
  if (nrows <= 0) return 0;
  cudaError_t e;
  {
    ProfScope p("block_offsets", stream);
    block_offsets_kernel<<<1, 32, 0, st>>>(a.cu_k, a.batch, a.blk_off);
  }
  e = cudaMemsetAsync(a.counts, 0, sizeof(int32_t) * a.nlists, st);
  if (e != cudaSuccess) return (int)e;
  e = cudaMemsetAsync(a.nitems, 0, sizeof(int32_t) * 2, st);   // nitems and the item ticket
  if (e != cudaSuccess) return (int)e;
  const int64_t nthreads = nrows * a.G;
  const int cs_blocks = (int)((nthreads + 255) / 256);
  {
    ProfScope p("count", stream);
    count_scatter_kernel<false><<<cs_blocks, 256, 0, st>>>(a.sel, a.t0, a.t1, a.G, a.k, a.batch, a.cu_q, a.cu_k,
                                                           a.blk_off, a.counts, nullptr, a.err);
  }
  {
    ProfScope p("plan", stream);
    plan_kernel<<<1, 1024, 0, st>>>(a.counts, a.nlists, a.G, a.batch, a.blk_off, a.queries_per_item, a.offsets,
                                    a.cursor, a.item_off, a.nitems, a.items, a.max_items, a.err);
  }
  {
    ProfScope p("scatter", stream);
    count_scatter_kernel<true><<<cs_blocks, 256, 0, st>>>(a.sel, a.t0, a.t1, a.G, a.k, a.batch, a.cu_q, a.cu_k,
                                                          a.blk_off, a.cursor, a.entries, a.err);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;

  alignas(64) CUtensorMap tm_k, tm_v;
  const uint64_t dims[3] = {(uint64_t)a.d, (uint64_t)a.G, (uint64_t)a.total_k};
  const uint64_t strides[2] = {(uint64_t)a.d * 2, (uint64_t)a.G * a.d * 2};
  const uint32_t box[3] = {64u, 1u, 128u};
  int rc = make_tmap_bf16(&tm_k, a.key, 3, dims, strides, box, 128);
  if (rc) return rc;
  rc = make_tmap_bf16(&tm_v, a.value, 3, dims, strides, box, 128);
  if (rc) return rc;
  const size_t smem = 1024 + (4 + kQSlots) * (size_t)128 * a.d * 2 + sizeof(AttnCtl);
  e = cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const float scale_log2 = a.sm_scale * 1.4426950408889634f;
  {
    ProfScope p("sparse_attn", stream);
    sparse_attn_kernel<<<nsm, kAttnThreads, smem, st>>>(
        tm_k, tm_v, reinterpret_cast<const __nv_bfloat16*>(a.q), a.items, a.nitems, a.nitems + 1, a.entries,
        a.cu_q, a.cu_k, a.H, a.G, a.d, a.k, scale_log2, a.t0, reinterpret_cast<__half*>(a.part_acc), a.part_lse,
        a.err);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  const int64_t rows = a.t1 - a.t0;
  const int64_t cthreads = rows * a.H * (a.d / 8);
  ProfScope p("combine", stream);
  combine_kernel<<<(int)((cthreads + 255) / 256), 256, 0, st>>>(
      reinterpret_cast<const __half*>(a.part_acc), a.part_lse, a.sel + a.t0 * a.G * a.k,
      reinterpret_cast<__nv_bfloat16*>(a.out) + a.t0 * a.H * a.d, a.lse ? a.lse + a.t0 * a.H : nullptr, rows, a.H,
      a.G, a.d, a.k);
  return (int)cudaGetLastError();
}

int launch_combine(const void* part_acc, const float* part_lse, const int32_t* sel, void* out, float* lse,
                   int64_t T, int32_t H, int32_t G, int32_t d, int32_t k, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T <= 0) return 0;
  const int64_t cthreads = T * H * (d / 8);
  ProfScope p("combine", stream);
  combine_kernel<<<(int)((cthreads + 255) / 256), 256, 0, st>>>(
      reinterpret_cast<const __half*>(part_acc), part_lse, sel, reinterpret_cast<__nv_bfloat16*>(out), lse, T, H, G,
      d, k);
  return (int)cudaGetLastError();
}

}  // namespace msa
