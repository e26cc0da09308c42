// Main Branch, KV-outer (pnsm.cn explainer sec. 7 "KV-outer sparse attention",
// "query gather", "two-phase combine"; yhxrc.cn sec. 二: loop over KV blocks and
// gather every query that chose the block, so each block is read once;
// yololab.net "KV Outer Gather Q").
//
// A pass over query rows [t0, t1):
//   0. tiles    : (msa_tile_attn.cu) the blocks that many queries of a small
//                 query tile share are marked for the query-tile kernel;
//   1. count    : per (group, window, sequence block) list, how many of the
//                 remaining (query, slot) entries chose it (warp-aggregated
//                 atomics);
//   2. plan     : exclusive scans -> list offsets, work items of at most
//                 `queries_per_item` queries per list;
//   3. scatter  : list entries (t - t0) * k + packed slot;
//   4. attend   : one work item = one KV block (TMA, loaded once) and up to
//                 queries_per_item gathered queries; per 128-row tile
//                 (128 / Hg queries x Hg heads) S = Q K^T and O = P V run on
//                 tcgen05 with fp32 accumulators in TMEM; each (query, group,
//                 block) writes its normalised output (f16) and log-sum-exp;
//      (the query-tile kernel then writes the shared blocks' results: final
//      outputs, or one merged partial per query)
//   5. combine  : per (query, head) log-sum-exp merge of the packed partials
//                 of every query on the combine list.
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

__global__ void block_offsets_kernel(const int32_t* __restrict__ cu_k, int batch, int B_k,
                                     int32_t* __restrict__ blk_off) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    int acc = 0;
    for (int b = 0; b < batch; ++b) {
      blk_off[b] = acc;
      acc += (cu_k[b + 1] - cu_k[b] + B_k - 1) / B_k;
    }
    blk_off[batch] = acc;
  }
}

// Validates an entry and returns its block's index over the whole batch
// (blk_off[b] + blk), or -1 (slot empty or invalid).
__device__ __forceinline__ int entry_block(int blk, int64_t t, int batch, int B_k, const int32_t* cu_q,
                                           const int32_t* cu_k, const int32_t* blk_off, DevError* err) {
  if (blk < 0) return -1;
  const int b = find_seq(cu_q, batch, t);
  const int Tb = cu_q[b + 1] - cu_q[b];
  const int Sb = cu_k[b + 1] - cu_k[b];
  const int64_t pos = (int64_t)Sb - Tb + (t - cu_q[b]);
  if (Tb > Sb || blk > pos / B_k) {
    report_error(err, MSA_ERR_DEVICE_CHECK, kSiteInvert, (int)t, blk);
    return -1;
  }
  return blk_off[b] + blk;
}

// Pass 1 and 3: one thread per (query, group).  Lists are keyed by
// (group, window of win_rows query rows, block): the work items come out
// group-major and, within a group, window by window, so the gathered rows of
// one group and window (win_rows x Hg x d x 2 bytes) stay hot in L2 while its
// items run, and consecutive windows of a group reuse that group's K/V blocks.
// kScatter == false counts, == true claims positions from `counter`
// (the cursors) and writes the entries (t - t0) * k + slot.
// Slots whose bit is set in dmask (when given) were attended by a query tile
// and get no list entry; they are still validated.  A pair's partials are
// packed at the front of its k-slot run: the tile's merged partial (if any)
// first, then its KV-outer slots in slot order, so that the combine reads one
// contiguous run per pair; an entry (t - t0) * k + p names packed position p.
// With clist (no query tiles), the counting pass also writes every pair's
// combine-list entry {pair, number of packed partials}.
template <bool kScatter>
__global__ void count_scatter_kernel(const int32_t* __restrict__ sel, int64_t t0, int64_t t1, int G, int k,
                                     int batch, int B_k, const int32_t* __restrict__ cu_q,
                                     const int32_t* __restrict__ cu_k,
                                     const int32_t* __restrict__ blk_off, int64_t nblocks, int64_t nwin,
                                     int win_rows, const uint32_t* __restrict__ dmask, int32_t* __restrict__ counter,
                                     uint32_t* __restrict__ entries, uint2* __restrict__ clist, DevError* err) {
  const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t n = (t1 - t0) * G;
  const bool active = gid < n;
  const int64_t tl = active ? gid / G : 0;
  const int64_t t = t0 + tl;
  const int g = active ? (int)(gid % G) : 0;
  const int64_t wbase = ((int64_t)g * nwin + tl / win_rows) * nblocks;
  const int lane = threadIdx.x & 31;
  const uint32_t covered = (active && dmask != nullptr) ? dmask[gid] : 0u;
  const int first = covered != 0u ? 1 : 0;   // packed position 0 holds the tile's merged partial
  uint32_t live = 0;                          // live slots below s
  for (int s = 0; s < k; ++s) {
    int64_t key = -1;
    int packed = 0;
    if (active) {
      const int32_t blk = sel[(t * G + g) * k + s];
      packed = first + __popc(live & ~covered);
      if (blk >= 0) live |= 1u << s;
      const int gb = entry_block(blk, t, batch, B_k, cu_q, cu_k, blk_off, err);
      if (gb >= 0 && !((covered >> s) & 1u)) key = wbase + gb;
    }
    // warp-aggregated atomics: lanes with the same key share one atomic
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    const int leader = __ffs(peers) - 1;
    const int rank = __popc(peers & ((1u << lane) - 1u));
    int base = 0;
    if (key >= 0 && lane == leader) base = atomicAdd(&counter[key], __popc(peers));
    base = __shfl_sync(0xffffffffu, base, leader);
    if (kScatter && key >= 0) entries[base + rank] = (uint32_t)(tl * k + packed);
  }
  if (!kScatter && clist != nullptr && active) clist[gid] = make_uint2((uint32_t)gid, (uint32_t)__popc(live));
}

// Device-wide exclusive scan of the list counts (and of their item counts,
// ceil(count / C)) in three passes over tiles of kScanTile keys.
constexpr int kScanThreads = 512;
constexpr int kScanPer = 8;
static_assert(kScanTile == kScanThreads * kScanPer, "scan tile");

__device__ __forceinline__ void block_scan2(int& a, int& b, int* sa, int* sb) {
  // inclusive scan of (a, b) over the block; sa/sb: 32-int shared scratch
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int ya = __shfl_up_sync(0xffffffffu, a, o), yb = __shfl_up_sync(0xffffffffu, b, o);
    if (lane >= o) { a += ya; b += yb; }
  }
  if (lane == 31) { sa[wid] = a; sb[wid] = b; }
  __syncthreads();
  if (wid == 0) {
    int wa = lane < kScanThreads / 32 ? sa[lane] : 0, wb = lane < kScanThreads / 32 ? sb[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ya = __shfl_up_sync(0xffffffffu, wa, o), yb = __shfl_up_sync(0xffffffffu, wb, o);
      if (lane >= o) { wa += ya; wb += yb; }
    }
    if (lane < kScanThreads / 32) { sa[lane] = wa; sb[lane] = wb; }
  }
  __syncthreads();
  if (wid > 0) { a += sa[wid - 1]; b += sb[wid - 1]; }
}

__global__ void __launch_bounds__(kScanThreads) scan_reduce_kernel(const int32_t* __restrict__ counts, int64_t nkeys,
                                                                  int C, int32_t* __restrict__ tile_sums) {
  __shared__ int sa[32], sb[32];
  const int64_t base = (int64_t)blockIdx.x * kScanTile + (int64_t)threadIdx.x * kScanPer;
  int a = 0, b = 0;
#pragma unroll
  for (int i = 0; i < kScanPer; ++i) {
    const int c = base + i < nkeys ? counts[base + i] : 0;
    a += c;
    b += (c + C - 1) / C;
  }
  block_scan2(a, b, sa, sb);
  if (threadIdx.x == kScanThreads - 1) {
    tile_sums[2 * blockIdx.x] = a;
    tile_sums[2 * blockIdx.x + 1] = b;
  }
}

// One CTA: exclusive scan of the tile sums (in place); totals -> nitems.
__global__ void __launch_bounds__(kScanThreads) scan_tiles_kernel(int32_t* __restrict__ tile_sums, int ntiles,
                                                                 int32_t* __restrict__ totals, int64_t max_items,
                                                                 DevError* err) {
  __shared__ int sa[32], sb[32];
  __shared__ int carry_a, carry_b;
  if (threadIdx.x == 0) { carry_a = 0; carry_b = 0; }
  __syncthreads();
  for (int base = 0; base < ntiles; base += kScanThreads) {
    const int i = base + threadIdx.x;
    const int a0 = i < ntiles ? tile_sums[2 * i] : 0, b0 = i < ntiles ? tile_sums[2 * i + 1] : 0;
    int a = a0, b = b0;
    block_scan2(a, b, sa, sb);
    const int ea = carry_a + a - a0, eb = carry_b + b - b0;
    if (i < ntiles) { tile_sums[2 * i] = ea; tile_sums[2 * i + 1] = eb; }
    __syncthreads();
    if (threadIdx.x == kScanThreads - 1) { carry_a = ea + a0; carry_b = eb + b0; }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const bool fits = carry_b <= max_items;
    totals[0] = fits ? carry_b : 0;      // items (the attention kernel's bound)
    totals[1] = 0;                       // item ticket
    totals[2] = carry_a;                 // entries
    if (!fits) report_error(err, MSA_ERR_WORKSPACE, kSiteInvert, carry_b, (int)max_items);
  }
}

// Final pass: list offsets and cursors, then the work items of each list
// (chunks of at most C entries), in key order (group-major, then window by window).
__global__ void __launch_bounds__(kScanThreads) scan_items_kernel(const int32_t* __restrict__ counts, int64_t nkeys,
                                                                 int64_t nblocks, int64_t nwin, int batch, int C,
                                                                 const int32_t* __restrict__ tile_sums,
                                                                 const int32_t* __restrict__ blk_off,
                                                                 int32_t* __restrict__ cursor,
                                                                 Item* __restrict__ items, int64_t max_items) {
  __shared__ int sa[32], sb[32];
  const int64_t base = (int64_t)blockIdx.x * kScanTile + (int64_t)threadIdx.x * kScanPer;
  int cnt[kScanPer];
  int a = 0, b = 0;
#pragma unroll
  for (int i = 0; i < kScanPer; ++i) {
    cnt[i] = base + i < nkeys ? counts[base + i] : 0;
    a += cnt[i];
    b += (cnt[i] + C - 1) / C;
  }
  int ia = a, ib = b;
  block_scan2(ia, ib, sa, sb);
  int off = tile_sums[2 * blockIdx.x] + ia - a;
  int io = tile_sums[2 * blockIdx.x + 1] + ib - b;
#pragma unroll
  for (int i = 0; i < kScanPer; ++i) {
    const int64_t key = base + i;
    if (key >= nkeys) break;
    cursor[key] = off;
    const int c = cnt[i];
    if (c > 0) {
      // key = (g * nwin + window) * nblocks + block of the batch
      const int gb = (int)(key % nblocks);
      const int g = (int)(key / (nblocks * nwin));
      int lo = 0, hi = batch;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (blk_off[mid] <= gb) lo = mid; else hi = mid;
      }
      for (int s = 0; s < c; s += C, ++io) {
        if (io >= max_items) break;
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
    off += c;
  }
}

// ------------------------------------------------------------ attention ---
//
// Warp-specialised, persistent (one CTA per SM, 512 threads):
//   warp 0      claims work items (atomic ticket) and publishes each one with
//               its query entries in a 4-deep shared-memory ring; lane 0 then
//               TMA-loads the item's K and V block into one of two stages and
//               gathers each 128-row tile's query rows with one TMA box per
//               (query, 64-column half) into one of three Q slots;
//   warp 1      owns TMEM (512 columns = two slots of S/P + O); its lane 0
//               issues every MMA, PV one tile behind S (S(t), PV(t-1), ...),
//               so the tensor core works on the next tile while tile t's
//               softmax runs (warps 2 and 3 are idle);
//   warps 4-7   softmax of even tiles (TMEM slot 0), warps 8-11 of odd tiles
//               (slot 1): S -> P (bf16, written back into the first 64 S
//               columns, the A operand of the PV MMA); each row's sum goes to
//               shared memory for the epilogue, its log-sum-exp to the partials;
//   warps 12-15 epilogue of every tile in order: O / l -> f16 partial and the
//               log-sum-exp of each row.
// A query occupies RQ = max(Hg, 8) tile rows (its Hg heads; with Hg = 4 the
// box also brings 4 rows of the next heads, which are ignored).

constexpr int kAttnThreads = 512;
constexpr int kItemRing = 4;
constexpr int kQSlots = 3;
constexpr int kItemEmptyCount = 13;   // MMA issuer 1 + softmax warps 8 + epilogue warps 4

struct __align__(16) RingItem {
  int32_t seq, blk, g, start, count, Tb, Sb, qrow0;
};

struct __align__(16) AttnCtl {
  uint64_t item_full[kItemRing], item_empty[kItemRing];
  uint64_t kv_full[2], kv_empty[2];
  uint64_t q_full[kQSlots], q_empty[kQSlots];
  uint64_t s_full[2], p_full[2], o_full[2], o_free[2];
  uint64_t stats_full[2];           // row sums of the slot's current tile are in row_sum
  uint64_t mma_done[2];
  uint32_t tmem_base;
  int32_t abort_flag;
  int32_t pad[2];
  RingItem ring[kItemRing];
  float row_sum[2][128];            // row sums of the unnormalised probabilities, per slot
};

__global__ void __launch_bounds__(kAttnThreads, 1)
sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_q, const Item* __restrict__ items,
                   const int32_t* __restrict__ nitems_p, int32_t* __restrict__ ticket,
                   const uint32_t* __restrict__ entries, const int32_t* __restrict__ cu_q,
                   const int32_t* __restrict__ cu_k, int H, int G, int d, int k, int B_k, float scale_log2,
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
  const int RQ = Hg < 8 ? 8 : Hg;              // tile rows per query
  const int qpt = 128 / RQ;                    // queries per 128-row tile
  const int nhalf = d / 64;
  const int nitems = *nitems_p;

  if (tid == 0) {
    for (int i = 0; i < kItemRing; ++i) { mbar_init(&ctl->item_full[i], 1); mbar_init(&ctl->item_empty[i], kItemEmptyCount); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->kv_full[i], 1); mbar_init(&ctl->kv_empty[i], 1);
      mbar_init(&ctl->s_full[i], 1); mbar_init(&ctl->p_full[i], 4);
      mbar_init(&ctl->o_full[i], 1); mbar_init(&ctl->o_free[i], 4);
      mbar_init(&ctl->stats_full[i], 4);
    }
    for (int i = 0; i < kQSlots; ++i) { mbar_init(&ctl->q_full[i], 1); mbar_init(&ctl->q_empty[i], 1); }
    mbar_init(&ctl->mma_done[0], 1);
    mbar_init(&ctl->mma_done[1], 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_q);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  // Waits for ring item n (consumers call this in the same order).
  // whole_warp: all 32 lanes call it (else only lane 0 of the warp does).
  auto wait_item = [&](int n) -> const RingItem* {
    const int slot = n % kItemRing;
    if (!mbar_wait(&ctl->item_full[slot], (n / kItemRing) & 1)) {
      report_error(err, MSA_ERR_TIMEOUT, kSiteAttnItem, n, warp);
      *abort_flag = 1;
      return nullptr;
    }
    return &ctl->ring[slot];
  };
  auto release_item = [&](int n, bool whole_warp) {
    if (whole_warp) __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->item_empty[n % kItemRing]);
  };

  if (warp == 0) {
    // ---------------------------------------- scheduler, K/V and Q loads
    int n = 0, tau = 0;
    while (true) {
      const int slot = n % kItemRing;
      bool ok = true;
      if (lane == 0) ok = mbar_wait(&ctl->item_empty[slot], ((n / kItemRing) + 1) & 1);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) {
        if (lane == 0) report_error(err, MSA_ERR_TIMEOUT, kSiteAttnLoad, n, 0);
        *abort_flag = 1;
        break;
      }
      int it = 0;
      if (lane == 0) it = *abort_flag ? nitems : atomicAdd(ticket, 1);
      it = __shfl_sync(0xffffffffu, it, 0);
      RingItem* R = &ctl->ring[slot];
      if (it >= nitems) {
        if (lane == 0) {
          R->count = 0;
          mbar_arrive(&ctl->item_full[slot]);
        }
        break;
      }
      const Item I = items[it];
      // this warp's lanes hold the item's entries (lane j: entries j, j + 32)
      const uint32_t e0 = lane < I.count ? entries[I.start + lane] : 0u;
      const uint32_t e1 = lane + 32 < I.count ? entries[I.start + lane + 32] : 0u;
      if (lane == 0) {
        R->seq = I.seq; R->blk = I.blk; R->g = I.g; R->start = I.start; R->count = I.count;
        R->Tb = cu_q[I.seq + 1] - cu_q[I.seq];
        R->Sb = cu_k[I.seq + 1] - cu_k[I.seq];
        R->qrow0 = cu_q[I.seq];
        mbar_arrive(&ctl->item_full[slot]);
        // K / V block of this item
        const int st = n & 1;
        ok = mbar_wait(&ctl->kv_empty[st], ((n >> 1) + 1) & 1);
        if (ok) {
          uint8_t* ks = kv_s + st * 2 * tile_bytes;
          mbar_arrive_expect_tx(&ctl->kv_full[st], 2 * tile_bytes);
          // the 128-row K/V tile starting at the block: B_k rows of it are the block
          const int krow = cu_k[I.seq] + I.blk * B_k;
          for (int h = 0; h < nhalf; ++h) {
            tma_load_3d(ks + h * 128 * 128, &tm_k, &ctl->kv_full[st], 64 * h, I.g, krow);
            tma_load_3d(ks + tile_bytes + h * 128 * 128, &tm_v, &ctl->kv_full[st], 64 * h, I.g, krow);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      // Q rows of each tile: lane ql issues the boxes of query ql
      const int ntiles = (I.count + qpt - 1) / qpt;
      for (int mt = 0; ok && mt < ntiles; ++mt, ++tau) {
        const int qs = tau % kQSlots;
        if (lane == 0) ok = mbar_wait(&ctl->q_empty[qs], ((tau / kQSlots) + 1) & 1);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        const int nq = min(qpt, I.count - mt * qpt);
        uint8_t* dst = q_s + qs * tile_bytes;
        if (lane == 0) mbar_arrive_expect_tx(&ctl->q_full[qs], nq * RQ * d * 2);
        __syncwarp();
        const int j = mt * qpt + lane;          // entry index of this lane's query
        const uint32_t ej = __shfl_sync(0xffffffffu, e0, j & 31);
        const uint32_t ek = __shfl_sync(0xffffffffu, e1, j & 31);
        if (lane < nq) {
          const int64_t t = t0 + (j < 32 ? ej : ek) / k;
          const int row = (int)(t * H + (int64_t)I.g * Hg);
          for (int h = 0; h < nhalf; ++h)
            tma_load_2d(dst + h * 128 * 128 + lane * RQ * 128, &tm_q, &ctl->q_full[qs], 64 * h, row);
        }
      }
      if (lane == 0 && !ok) {
        report_error(err, MSA_ERR_TIMEOUT, kSiteAttnLoad, n, 1);
        *abort_flag = 1;
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      ++n;
    }
    if (lane == 0) {
      // no TMA load may still be in flight when the CTA exits
      for (int st = 0; st < 2; ++st) {
        const int issued = n > st ? (n - st + 1) / 2 : 0;
        if (issued > 0) mbar_wait(&ctl->kv_full[st], (issued - 1) & 1);
      }
      for (int qs = 0; qs < kQSlots; ++qs) {
        const int issued = tau > qs ? (tau - qs + kQSlots - 1) / kQSlots : 0;
        if (issued > 0) mbar_wait(&ctl->q_full[qs], (issued - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    // One thread issues every MMA, one tile behind for PV: S(t), PV(t-1),
    // S(t+1), PV(t), ...  tcgen05.mma operations of one thread run in issue
    // order, so S(t) may overwrite slot t%2, whose first 64 columns hold the
    // P(t-2) that PV(t-2) read, as soon as PV(t-2) has been issued.
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t idesc_o = idesc_bf16_f32(128, d, 0, 1);
      // descriptors built once; per-slot / per-step byte offsets (>> 4) are added
      const uint64_t qdesc0 = make_sdesc(smem_u32(q_s), 16, 1024, kSw128);
      const uint64_t kvdesc0 = make_sdesc(smem_u32(kv_s), 16, 1024, kSw128);
      const uint64_t vdesc0 = make_sdesc(smem_u32(kv_s + tile_bytes), 128 * 128, 1024, kSw128);
      int n = 0, tau = 0;
      bool ok = true;
      bool pend = false, pend_last = false;     // PV of tile tau-1 not yet issued
      int pend_st = 0;
      // PV of tile t (K/V stage st); the item's last tile releases the stage
      auto issue_pv = [&](int t, int st, bool last) -> bool {
        const int s = t & 1;
        if (!mbar_wait(&ctl->p_full[s], (t >> 1) & 1) || !mbar_wait(&ctl->o_free[s], ((t >> 1) + 1) & 1))
          return false;
        tc_fence_after();
        const uint64_t vd = vdesc0 + (uint64_t)((st * 2 * tile_bytes) >> 4);
        const uint32_t pcol = tmem + s * 256, ocol = pcol + 128;
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16_ts(ocol, pcol + kk * 8, vd + (uint64_t)((kk * 2048) >> 4), idesc_o, kk > 0 ? 1u : 0u);
        umma_commit(&ctl->o_full[s]);
        if (last) umma_commit(&ctl->kv_empty[st]);
        return true;
      };
      while (ok && !*abort_flag) {
        const RingItem* R = wait_item(n);
        if (R == nullptr) { ok = false; break; }
        const int cnt = R->count;
        release_item(n, false);
        if (cnt <= 0) break;
        const int st = n & 1;
        const int ntiles = (cnt + qpt - 1) / qpt;
        for (int mt = 0; mt < ntiles && ok; ++mt, ++tau) {
          const int s = tau & 1;
          const int qs = tau % kQSlots;
          if (!mbar_wait(&ctl->q_full[qs], (tau / kQSlots) & 1) ||
              (mt == 0 && !mbar_wait(&ctl->kv_full[st], (n >> 1) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t qd = qdesc0 + (uint64_t)((qs * tile_bytes) >> 4);
          const uint64_t kd = kvdesc0 + (uint64_t)((st * 2 * tile_bytes) >> 4);
          for (int kk = 0; kk < d / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4);
            umma_bf16_ss(tmem + s * 256, qd + off, kd + off, idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(&ctl->s_full[s]);
          umma_commit(&ctl->q_empty[qs]);
          if (pend && !issue_pv(tau - 1, pend_st, pend_last)) {
            ok = false;
            break;
          }
          pend = true;
          pend_st = st;
          pend_last = (mt == ntiles - 1);
        }
        ++n;
      }
      if (ok && pend && !issue_pv(tau - 1, pend_st, pend_last)) ok = false;
      if (!ok) {
        report_error(err, MSA_ERR_TIMEOUT, kSiteAttnMma, tau, 0);
        *abort_flag = 1;
      }
      umma_commit(&ctl->mma_done[0]);
      mbar_wait(&ctl->mma_done[0], 0);
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ softmax
    const int wg = (warp - 4) >> 2;           // slot handled by this warpgroup
    const int wq = warp & 3;                  // TMEM lane quarter
    const int r = 32 * wq + lane;             // tile row
    const uint32_t s_col = tmem + wg * 256 + (static_cast<uint32_t>(32 * wq) << 16);   // S, then P
    const int ql = r / RQ, hi = r - ql * RQ;
    int n = 0, tau = 0;
    while (!*abort_flag) {
      const RingItem* R = wait_item(n);
      if (R == nullptr) break;
      const int count = R->count;
      if (count <= 0) { release_item(n, true); break; }
      const int Tb = R->Tb, Sb = R->Sb;
      const int64_t qrow0 = R->qrow0;
      const int64_t blk_first = (int64_t)R->blk * B_k;
      const int ntiles = (count + qpt - 1) / qpt;
      // the item stays in the ring until this warpgroup's last tile of it
      for (int mt = 0; mt < ntiles; ++mt, ++tau) {
        if ((tau & 1) != wg) continue;
        const int idx = mt * qpt + ql;
        const bool valid = ql < qpt && idx < count && hi < Hg;
        const uint32_t e = valid ? entries[R->start + idx] : 0u;
        // last attended key of the tile: the block's last (B_k - 1), or the causal cut
        int limit = B_k - 1;
        if (valid) {
          const int64_t t = t0 + e / k;
          const int64_t lim = (int64_t)Sb - Tb + (t - qrow0) - blk_first;
          limit = lim >= B_k - 1 ? B_k - 1 : (int)lim;
        }
        if (!mbar_wait(&ctl->s_full[wg], (tau >> 1) & 1)) {
          report_error(err, MSA_ERR_TIMEOUT, kSiteAttnSoftmax, tau, 0);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        uint32_t rr[32];
        float m = -INFINITY, l = 0.f, ms;
        if (__all_sync(0xffffffffu, limit >= 127)) {
          // no causal cut in this warp's rows (not the local block)
#pragma unroll 1
          for (int c4 = 0; c4 < 4; ++c4) {
            tmem_ld32(s_col + 32 * c4, rr);
            tmem_ld_wait();
            float mm[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) mm[j] = fmaxf(__uint_as_float(rr[2 * j]), __uint_as_float(rr[2 * j + 1]));
#pragma unroll
            for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
              for (int j = 0; j < w; ++j) mm[j] = fmaxf(mm[j], mm[j + w]);
            m = fmaxf(m, mm[0]);
          }
          ms = m * scale_log2;
#pragma unroll 1
          for (int c4 = 0; c4 < 4; ++c4) {
            tmem_ld32(s_col + 32 * c4, rr);
            tmem_ld_wait();
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float p0 = ex2_approx(fmaf(__uint_as_float(rr[2 * j]), scale_log2, -ms));
              const float p1 = ex2_approx(fmaf(__uint_as_float(rr[2 * j + 1]), scale_log2, -ms));
              l += p0 + p1;
              pk[j] = pack_bf16x2(p0, p1);
            }
            tmem_st16(s_col + 16 * c4, pk);
          }
        } else {
#pragma unroll 1
          for (int c4 = 0; c4 < 4; ++c4) {
            tmem_ld32(s_col + 32 * c4, rr);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j)
              m = fmaxf(m, 32 * c4 + j <= limit ? __uint_as_float(rr[j]) : -INFINITY);
          }
          ms = m * scale_log2;
#pragma unroll 1
          for (int c4 = 0; c4 < 4; ++c4) {
            tmem_ld32(s_col + 32 * c4, rr);
            tmem_ld_wait();
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int c0 = 32 * c4 + 2 * j;
              const float x0 = fmaf(__uint_as_float(rr[2 * j]), scale_log2, -ms);
              const float x1 = fmaf(__uint_as_float(rr[2 * j + 1]), scale_log2, -ms);
              const float p0 = ex2_approx(c0 <= limit ? x0 : -INFINITY);
              const float p1 = ex2_approx(c0 + 1 <= limit ? x1 : -INFINITY);
              l += p0 + p1;
              pk[j] = pack_bf16x2(p0, p1);
            }
            tmem_st16(s_col + 16 * c4, pk);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->p_full[wg]);
        if (valid) {
          const int64_t unit = ((int64_t)(e / k) * G + R->g) * k + (e % k);
          // write-once data: streaming stores (evict-first in L2), which keep the
          // window's gathered Q rows resident
          __stcs(part_lse + unit * Hg + hi, (ms + __log2f(l)) * 0.69314718055994530942f);
        }
        // the epilogue of tile tau-2 (same slot) has read row_sum[wg] once o_free fires
        if (!mbar_wait(&ctl->o_free[wg], ((tau >> 1) + 1) & 1)) {
          report_error(err, MSA_ERR_TIMEOUT, kSiteAttnSoftmax, tau, 2);
          *abort_flag = 1;
          break;
        }
        ctl->row_sum[wg][r] = l;
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->stats_full[wg]);
      }
      release_item(n, true);
      ++n;
    }
  } else if (warp >= 12) {
    // ----------------------------------------------------------- epilogue
    const int wq = warp & 3;                  // TMEM lane quarter
    const int r = 32 * wq + lane;             // tile row
    const uint32_t lane_off = static_cast<uint32_t>(32 * wq) << 16;
    const int ql = r / RQ, hi = r - ql * RQ;
    int n = 0, tau = 0;
    while (!*abort_flag) {
      const RingItem* R = wait_item(n);
      if (R == nullptr) break;
      const int count = R->count, g = R->g;
      if (count <= 0) { release_item(n, true); break; }
      const int ntiles = (count + qpt - 1) / qpt;
      for (int mt = 0; mt < ntiles; ++mt, ++tau) {
        const int s = tau & 1;
        const int idx = mt * qpt + ql;
        const bool valid = ql < qpt && idx < count && hi < Hg;
        const uint32_t e = valid ? entries[R->start + idx] : 0u;
        if (!mbar_wait(&ctl->stats_full[s], (tau >> 1) & 1) || !mbar_wait(&ctl->o_full[s], (tau >> 1) & 1)) {
          report_error(err, MSA_ERR_TIMEOUT, kSiteAttnSoftmax, tau, 1);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const float inv_l = 1.f / ctl->row_sum[s][r];
        const int64_t unit = valid ? ((int64_t)(e / k) * G + g) * k + (e % k) : 0;
        // partial layout per unit: [d/8 chunks][Hg heads][8 values], so the
        // 16 heads of one query write 256 contiguous bytes per chunk
        __half* dst = part_acc + unit * Hg * d + hi * 8;
        const uint32_t o_col = tmem + s * 256 + 128 + lane_off;
        uint32_t rr[32];
#pragma unroll 1
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
              __stcs(reinterpret_cast<uint4*>(dst + (4 * c4 + j) * Hg * 8), w);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->o_free[s]);
      }
      release_item(n, true);
      ++n;
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

// Persistent combine.  The partials of one (query, group) are one contiguous
// run (k slots x [d/8][Hg][8] f16, 4 KB per slot at Hg = 16, d = 128), its
// k x Hg log-sum-exps another.  A chunk is P (query, group) pairs, handled by
// one consumer group of 256 threads: thread (pair, c, i) merges output columns
// 8c..8c+7 of head i (a pair spans Hg * d/8 threads, a multiple of 32;
// consecutive threads read consecutive 16-byte words of shared memory).
//   clist given: entry {pair, n} per merged pair, partials packed in slots
//                0..n-1: only those n slots are copied (the query tiles leave
//                most slots empty);
//   clist null : every pair, slots with sel >= 0, whole runs copied.
// Warp 16 (lane 0) is the producer: it streams each chunk's runs with bulk
// async copies into a byte-granular ring of shared memory (a chunk takes what
// its runs need, so the bytes in flight follow the real sizes) and publishes
// it in a queue of kCombQueue entries; consumer groups 0 and 1 take alternate
// entries and release them through per-entry barriers, so the two groups and
// the producer never wait for one another except on data.
constexpr int kCombGroupThreads = 256;
constexpr int kCombThreads = 2 * kCombGroupThreads + 32;
constexpr int kCombQueue = 8;
constexpr int kCombMaxPairs = 8;
constexpr uint32_t kCombRing = 200 * 1024;

struct CombEntry {
  uint32_t off[kCombMaxPairs];   // ring offset of each pair's run (partials, then log-sum-exps)
  uint32_t pair[kCombMaxPairs];
  uint32_t n[kCombMaxPairs];     // slots copied
};

struct CombCtl {
  uint64_t full[kCombQueue], consumed[kCombQueue];
  uint64_t end_of[kCombQueue];   // producer: virtual ring offset after each entry
  CombEntry e[kCombQueue];
  int32_t abort_flag;
};

__global__ void __launch_bounds__(kCombThreads, 1)
combine_kernel(const __half* __restrict__ part_acc, const float* __restrict__ part_lse,
               const int32_t* __restrict__ sel, const uint2* __restrict__ clist,
               const int32_t* __restrict__ npairs_dev, __nv_bfloat16* __restrict__ out, float* __restrict__ lse_out,
               int64_t T, int H, int G, int d, int k, int P, uint32_t acc_bytes, uint32_t lse_bytes,
               DevError* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* ring = smem_raw + (((raw + 127u) & ~127u) - raw);
  __shared__ CombCtl ctl;
  volatile int32_t* abort_flag = &ctl.abort_flag;
  const int Hg = H / G;
  const int per = Hg * (d / 8);                 // threads per (query, group)
  const uint32_t slot_bytes = acc_bytes / k;    // one slot's partial (multiple of 16)
  const uint32_t slot_lse = lse_bytes / k;      // one slot's Hg log-sum-exps (multiple of 16)
  const int64_t npairs = npairs_dev != nullptr ? (int64_t)*npairs_dev : T * G;
  const int64_t nchunks = (npairs + P - 1) / P;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < kCombQueue; ++i) {
      mbar_init(&ctl.full[i], 1);
      mbar_init(&ctl.consumed[i], kCombGroupThreads / 32);
    }
    ctl.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // the m-th chunk of this CTA is chunk blockIdx.x + m * gridDim.x
  const int64_t my = blockIdx.x < nchunks ? (nchunks - 1 - blockIdx.x) / gridDim.x + 1 : 0;

  if (warp == 2 * kCombGroupThreads / 32) {
    // ------------------------------------------------------------ producer
    // The whole warp loads the list entries of 32 chunks ahead (lane l: chunk
    // m0 + l); lane 0 allocates ring space, waits and issues the copies.
    auto load_batch = [&](int64_t m0, uint2 (&dst)[kCombMaxPairs]) {
      const int64_t mm = m0 + lane;
      const int64_t p0 = (blockIdx.x + mm * gridDim.x) * P;
#pragma unroll
      for (int i = 0; i < kCombMaxPairs; ++i) {
        dst[i] = make_uint2(0u, 0u);
        if (i < P && mm < my && p0 + i < npairs)
          dst[i] = clist != nullptr ? clist[p0 + i] : make_uint2((uint32_t)(p0 + i), (uint32_t)k);
      }
    };
    uint2 cur[kCombMaxPairs], nxt[kCombMaxPairs];
    load_batch(0, cur);
    load_batch(32, nxt);
    uint64_t alloc = 0, freed = 0;              // virtual ring offsets (physical = virtual % ring)
    int64_t oldest = 0, m = 0, issued = 0;      // issued: chunks whose copies were started (lane 0)
    bool ok = true;
    for (; m < my; ++m) {
      bool go = lane == 0 ? (ok && !*abort_flag) : true;
      go = __shfl_sync(0xffffffffu, go ? 1 : 0, 0) != 0;
      if (!go) break;
      if (m > 0 && (m & 31) == 0) {
#pragma unroll
        for (int i = 0; i < kCombMaxPairs; ++i) cur[i] = nxt[i];
        load_batch(m + 32, nxt);
      }
      uint2 ent[kCombMaxPairs];
#pragma unroll
      for (int i = 0; i < kCombMaxPairs; ++i) {
        ent[i].x = __shfl_sync(0xffffffffu, cur[i].x, (int)(m & 31));
        ent[i].y = __shfl_sync(0xffffffffu, cur[i].y, (int)(m & 31));
      }
      if (lane != 0) continue;
      const int q = (int)(m % kCombQueue);
      const int64_t p0 = (blockIdx.x + m * gridDim.x) * P;
      const int np = npairs - p0 < P ? (int)(npairs - p0) : P;
      uint32_t bytes = 0;
#pragma unroll
      for (int i = 0; i < kCombMaxPairs; ++i)
        if (i < np) bytes += ent[i].y * (slot_bytes + slot_lse);
      // contiguous room in the ring (skip the ring's tail end when it is too short)
      const uint64_t phys = alloc % kCombRing;
      if (phys + bytes > kCombRing) alloc += kCombRing - phys;
      // the queue entry and the bytes must both be free: retire the oldest entries in order
      while (ok && (m - oldest >= kCombQueue || alloc + bytes - freed > kCombRing)) {
        if (oldest == m) {                      // nothing in flight: the whole ring is free
          freed = alloc;
          continue;
        }
        const int qo = (int)(oldest % kCombQueue);
        ok = mbar_wait(&ctl.consumed[qo], (uint32_t)((oldest / kCombQueue) & 1));
        if (ok) { freed = ctl.end_of[qo]; ++oldest; }
      }
      if (!ok) continue;                        // the next iteration's check ends the loop
      // entry q is free (its previous chunk was consumed): publish this chunk in it
      CombEntry& E = ctl.e[q];
      uint32_t off = (uint32_t)(alloc % kCombRing);
      mbar_arrive_expect_tx(&ctl.full[q], bytes);
#pragma unroll
      for (int i = 0; i < kCombMaxPairs; ++i) {
        if (i >= np) continue;
        E.off[i] = off;
        E.pair[i] = ent[i].x;
        E.n[i] = ent[i].y;
        const uint32_t na = ent[i].y * slot_bytes, nl = ent[i].y * slot_lse;
        bulk_load(ring + off, reinterpret_cast<const uint8_t*>(part_acc) + (int64_t)ent[i].x * acc_bytes, na,
                  &ctl.full[q]);
        bulk_load(ring + off + na, reinterpret_cast<const uint8_t*>(part_lse) + (int64_t)ent[i].x * lse_bytes, nl,
                  &ctl.full[q]);
        off += na + nl;
      }
      alloc += bytes;
      ctl.end_of[q] = alloc;
      issued = m + 1;
    }
    if (lane == 0) {
      if (!ok) {
        report_error(err, MSA_ERR_TIMEOUT, kSiteAttnLoad, (int)m, -2);
        *abort_flag = 1;
      }
      // no bulk copy may still be writing when the CTA exits
      for (int64_t j = oldest; j < issued; ++j) mbar_wait(&ctl.full[j % kCombQueue], (uint32_t)((j / kCombQueue) & 1));
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int grp = warp / (kCombGroupThreads / 32);
  const int gt = tid - grp * kCombGroupThreads;
  const int pl = gt / per;                      // pair within the chunk (P * per == kCombGroupThreads)
  const int rem = gt - pl * per;
  const int cc = rem / Hg, i = rem - cc * Hg;
  for (int64_t m = grp; m < my && !*abort_flag; m += 2) {
    const int q = (int)(m % kCombQueue);
    const int64_t idx = (blockIdx.x + m * gridDim.x) * P + pl;
    const bool live = idx < npairs;
    uint32_t valid = 0;
    if (clist == nullptr) {
      const int32_t sv = (lane < k && live) ? __ldg(sel + idx * k + lane) : -1;
      valid = __ballot_sync(0xffffffffu, sv >= 0);
    }
    if (!mbar_wait(&ctl.full[q], (uint32_t)((m / kCombQueue) & 1))) {
      report_error(err, MSA_ERR_TIMEOUT, kSiteAttnLoad, (int)m, -3);
      *abort_flag = 1;
      break;
    }
    if (live) {
      const CombEntry& E = ctl.e[q];
      const int n = (int)E.n[pl];
      const int64_t pair = E.pair[pl];
      if (clist != nullptr) valid = n >= 32 ? 0xffffffffu : (1u << n) - 1u;
      const __half* acc_s = reinterpret_cast<const __half*>(ring + E.off[pl]);
      const float* lse_s = reinterpret_cast<const float*>(ring + E.off[pl] + n * slot_bytes);
      float m_ = -INFINITY;
#pragma unroll 4
      for (int s2 = 0; s2 < n; ++s2)
        if ((valid >> s2) & 1u) m_ = fmaxf(m_, lse_s[s2 * Hg + i]);
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      float wsum = 0.f;
#pragma unroll 4
      for (int s2 = 0; s2 < n; ++s2) {
        // an unused slot is skipped, not weighted by 0: its buffer may hold anything (NaN included)
        if (!((valid >> s2) & 1u)) continue;
        const float w = __expf(lse_s[s2 * Hg + i] - m_);
        wsum += w;
        const uint4 rv = *reinterpret_cast<const uint4*>(acc_s + ((s2 * (d / 8) + cc) * Hg + i) * 8);
        const __half2* hp = reinterpret_cast<const __half2*>(&rv);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __half22float2(hp[j]);
          acc[2 * j] = fmaf(w, f.x, acc[2 * j]);
          acc[2 * j + 1] = fmaf(w, f.y, acc[2 * j + 1]);
        }
      }
      const float inv = 1.f / wsum;
      uint4 o;
      o.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
      o.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
      o.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
      o.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
      const int64_t t = pair / G;
      const int h = (int)(pair - t * G) * Hg + i;
      __stcs(reinterpret_cast<uint4*>(out + (t * H + h) * d + 8 * cc), o);
      if (lse_out != nullptr && cc == 0) __stcs(lse_out + t * H + h, m_ + __logf(wsum));
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl.consumed[q]);
  }
}

int launch_combine_kernel(const __half* part_acc, const float* part_lse, const int32_t* sel, const uint2* clist,
                          const int32_t* npairs_dev, __nv_bfloat16* out, float* lse, int64_t T, int H, int G, int d,
                          int k, DevError* err, cudaStream_t st, int grid_cap = 0) {
  if (T <= 0) return 0;
  const int Hg = H / G;
  const int per = Hg * (d / 8);
  if (per % 32 != 0 || kCombGroupThreads % per != 0 || k > 32) return (int)cudaErrorInvalidValue;
  const int P = kCombGroupThreads / per;
  if (P > kCombMaxPairs) return (int)cudaErrorInvalidValue;
  const uint32_t acc_bytes = (uint32_t)k * Hg * d * 2;
  const uint32_t lse_bytes = (uint32_t)k * Hg * 4;
  // bulk copies need 16-byte sizes and addresses; one chunk must fit the ring
  if (((acc_bytes / k | lse_bytes / k) & 15u) || ((reinterpret_cast<uintptr_t>(part_acc) |
                                                   reinterpret_cast<uintptr_t>(part_lse)) & 15u) ||
      (uint64_t)P * (acc_bytes + lse_bytes) > kCombRing)
    return (int)cudaErrorInvalidValue;
  const size_t smem = 128 + kCombRing;
  cudaError_t e = cudaFuncSetAttribute(combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int64_t nchunks = (T * G + P - 1) / P;   // upper bound when a list is given
  const int cap = grid_cap > 0 && grid_cap < nsm ? grid_cap : nsm;
  const int grid = (int)(nchunks < cap ? nchunks : cap);
  combine_kernel<<<grid, kCombThreads, smem, st>>>(part_acc, part_lse, sel, clist, npairs_dev, out, lse, T, H, G, d,
                                                  k, P, acc_bytes, lse_bytes, err);
  return (int)cudaGetLastError();
}

}  // namespace

// -------------------------------------------------------------- launchers ---

int launch_kv_plan(const AttnArgs& a, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t nrows = a.t1 - a.t0;
  if (nrows <= 0) return 0;
  cudaError_t e;
  {
    ProfScope p("block_offsets", stream);
    block_offsets_kernel<<<1, 32, 0, st>>>(a.cu_k, a.batch, a.B_k, a.blk_off);
  }
  const int win = a.win_rows;
  const int64_t nwin = (nrows + win - 1) / win;
  const int64_t nkeys = nwin * a.nlists;
  const int64_t nblocks = a.nlists / a.G;
  e = cudaMemsetAsync(a.counts, 0, sizeof(int32_t) * nkeys, st);
  if (e != cudaSuccess) return (int)e;
  const bool tiles = a.theta > 0;
  if (tiles) {
    e = cudaMemsetAsync(a.tile_ctr, 0, sizeof(int32_t) * 4, st);
    if (e != cudaSuccess) return (int)e;
    const int rc = launch_tile_plan(a, a.theta, stream);
    if (rc) return rc;
  }
  const uint32_t* dmask = tiles ? a.dmask : nullptr;
  const int64_t nthreads = nrows * a.G;
  const int cs_blocks = (int)((nthreads + 255) / 256);
  {
    ProfScope p("count", stream);
    count_scatter_kernel<false><<<cs_blocks, 256, 0, st>>>(a.sel, a.t0, a.t1, a.G, a.k, a.batch, a.B_k, a.cu_q, a.cu_k,
                                                           a.blk_off, nblocks, nwin, win, dmask, a.counts, nullptr,
                                                           tiles ? nullptr : a.clist, a.err);
  }
  const int ntiles = (int)((nkeys + kScanTile - 1) / kScanTile);
  {
    ProfScope p("plan", stream);
    scan_reduce_kernel<<<ntiles, kScanThreads, 0, st>>>(a.counts, nkeys, a.queries_per_item, a.tile_sums);
    scan_tiles_kernel<<<1, kScanThreads, 0, st>>>(a.tile_sums, ntiles, a.nitems, a.max_items, a.err);
    scan_items_kernel<<<ntiles, kScanThreads, 0, st>>>(a.counts, nkeys, nblocks, nwin, a.batch, a.queries_per_item,
                                                       a.tile_sums, a.blk_off, a.cursor, a.items, a.max_items);
    prof_count_launch(2);
  }
  {
    ProfScope p("scatter", stream);
    count_scatter_kernel<true><<<cs_blocks, 256, 0, st>>>(a.sel, a.t0, a.t1, a.G, a.k, a.batch, a.B_k, a.cu_q, a.cu_k,
                                                          a.blk_off, nblocks, nwin, win, dmask, a.cursor, a.entries,
                                                          nullptr,
                                                          a.err);
  }
  return (int)cudaGetLastError();
}

int launch_sparse_attn_main(const AttnArgs& a, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (a.t1 - a.t0 <= 0) return 0;
  int rc0 = launch_kv_plan(a, stream);
  if (rc0) return rc0;
  const bool tiles = a.theta > 0;
  cudaError_t e;

  alignas(64) CUtensorMap tm_k, tm_v, tm_q;
  {
    const uint64_t dims[3] = {(uint64_t)a.d, (uint64_t)a.G, (uint64_t)a.total_k};
    const uint64_t strides[2] = {(uint64_t)a.d * 2, (uint64_t)a.G * a.d * 2};
    const uint32_t box[3] = {64u, 1u, 128u};
    int rc = make_tmap_bf16(&tm_k, a.key, 3, dims, strides, box, 128);
    if (rc) return rc;
    rc = make_tmap_bf16(&tm_v, a.value, 3, dims, strides, box, 128);
    if (rc) return rc;
  }
  {
    const int hg = a.H / a.G;
    const uint64_t dims[2] = {(uint64_t)a.d, (uint64_t)a.total_q * a.H};
    const uint64_t strides[1] = {(uint64_t)a.d * 2};
    const uint32_t box[2] = {64u, (uint32_t)(hg < 8 ? 8 : hg)};
    int rc = make_tmap_bf16(&tm_q, a.q, 2, dims, strides, box, 128);
    if (rc) return rc;
  }
  const size_t smem = 1024 + (4 + kQSlots) * (size_t)128 * a.d * 2 + sizeof(AttnCtl);
  static_assert(1024 + 7 * 128 * 128 * 2 + sizeof(AttnCtl) <= 227 * 1024, "shared memory budget (d = 128)");
  e = cudaFuncSetAttribute(sparse_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const float scale_log2 = a.sm_scale * 1.4426950408889634f;
  {
    ProfScope p("sparse_attn", stream);
    sparse_attn_kernel<<<nsm, kAttnThreads, smem, st>>>(
        tm_k, tm_v, tm_q, a.items, a.nitems, a.nitems + 1, a.entries, a.cu_q, a.cu_k, a.H, a.G, a.d, a.k, a.B_k,
        scale_log2, a.t0, reinterpret_cast<__half*>(a.part_acc), a.part_lse, a.err);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  if (tiles) {
    const int rc = launch_tile_attn(a, stream);
    if (rc) return rc;
  }
  return 0;
}

int launch_sparse_attn_combine(const AttnArgs& a, void* stream, int grid_cap) {
  const int64_t rows = a.t1 - a.t0;
  if (rows <= 0) return 0;
  ProfScope p("combine", stream);
  return launch_combine_kernel(reinterpret_cast<const __half*>(a.part_acc), a.part_lse, a.sel + a.t0 * a.G * a.k,
                               a.clist, a.theta > 0 ? a.tile_ctr : nullptr,
                               reinterpret_cast<__nv_bfloat16*>(a.out) + a.t0 * a.H * a.d,
                               a.lse ? a.lse + a.t0 * a.H : nullptr, rows, a.H, a.G, a.d, a.k, a.err,
                               reinterpret_cast<cudaStream_t>(stream), grid_cap);
}

int launch_sparse_attn_pass(const AttnArgs& a, void* stream) {
  const int rc = launch_sparse_attn_main(a, stream);
  return rc ? rc : launch_sparse_attn_combine(a, stream, 0);
}

int launch_combine(const void* part_acc, const float* part_lse, const int32_t* sel, void* out, float* lse,
                   int64_t T, int32_t H, int32_t G, int32_t d, int32_t k, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T <= 0) return 0;
  ProfScope p("combine", stream);
  return launch_combine_kernel(reinterpret_cast<const __half*>(part_acc), part_lse, sel, nullptr, nullptr,
                               reinterpret_cast<__nv_bfloat16*>(out), lse, T, H, G, d, k, nullptr, st);
}

}  // namespace msa
