// Index Branch, prefill shape: raw index scores on tcgen05, block max-pooling in
// the TMEM epilogue, and a per-thread register top-(k-1) with the forced local
// block (pnsm.cn explainer sec. 2 and sec. 7 "exp-free Top-k" / "per-thread
// register top-k"; yifor-blog "設計核心" item 1; yhxrc.cn sec. 二 "block max
// pooling").
//
// One persistent CTA per SM walks work units = (128-query tile, pair of GQA
// groups); the two groups of a unit share each index-key block load.  Per key
// block j the tensor core computes S_g = Q_idx[g][128 x d_idx] * K_idx[j]^T for
// both groups into one of two TMEM buffers (2 buffers x 2 groups x 128 columns),
// so the epilogue drains block j while block j+1 is being computed.  An
// epilogue warpgroup per group reads its lane's 128 scores, takes the max (the
// block score) and offers (score, j) to the register top list of that
// (query, group).  Blocks arrive in ascending order, so a new block only
// displaces a strictly lower score: ties stay with the lower block index.
//
// Warp roles (352 threads): warps 4l .. 4l+3 are the epilogue of the unit's
// l-th group, warp 8 issues TMA loads, warp 9 owns TMEM, and lane 0 of warp
// 9 + l issues the MMAs of group l.  One issuing thread per group: a thread
// that interleaves tcgen05.commit with its MMAs issues at about half the MMA
// rate, so each group gets its own issue and commit stream.
#include "msa_common.cuh"

namespace msa {
namespace {

constexpr int kStages = 6;        // max index-key block stages in shared memory
constexpr int kThreads = 352;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;     // and kMmaWarp + 1 for the second group of a pair
constexpr int kTile = 128;        // queries per tile = key-block size

struct __align__(16) IndexCtl {
  uint64_t q_full, q_empty;
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t acc_full[2][2], acc_empty[2][2];   // [buffer][group slot]
  uint64_t mma_done[2];
  uint32_t tmem_base;
  int32_t abort_flag;
  int32_t ntiles;             // tiles of this launch: tau0 .. tau0 + ntiles - 1
  int32_t tau0;
  int32_t tile_prefix[kMaxBatchTiles + 1];
};

struct TileInfo {
  int q0;      // first query row of the tile
  int rows;    // valid query rows (<= 128)
  int pos0;    // absolute position of row 0 in its sequence
  int n_kb;    // 128-key tiles scanned: 0 .. n_kb-1 (they hold the blocks before the last row's local block)
  int k0row;   // first key row of the sequence
};

__device__ __forceinline__ TileInfo tile_info(int tau, const IndexCtl* ctl, int batch, const int32_t* cu_q,
                                              const int32_t* cu_k, int B_k) {
  int lo = 0, hi = batch;  // find b with prefix[b] <= tau < prefix[b+1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (ctl->tile_prefix[mid] <= tau) lo = mid; else hi = mid;
  }
  const int b = lo;
  const int i = tau - ctl->tile_prefix[b];
  const int Tb = cu_q[b + 1] - cu_q[b];
  const int Sb = cu_k[b + 1] - cu_k[b];
  TileInfo t;
  t.q0 = cu_q[b] + kTile * i;
  t.rows = min(kTile, Tb - kTile * i);
  t.pos0 = Sb - Tb + kTile * i;
  t.n_kb = ((t.pos0 + t.rows - 1) / B_k * B_k + kBk - 1) / kBk;
  t.k0row = cu_k[b];
  return t;
}

// Static snake schedule over work units in longest-first order: iteration
// `it` of CTA c takes slot it*grid + (it even ? c : grid-1-c); slot s is unit
// nunits-1-s (units of later tiles scan more key blocks).
__device__ __forceinline__ int snake_unit(int it, int nunits) {
  const int g = gridDim.x, c = blockIdx.x;
  const int slot = it * g + ((it & 1) ? (g - 1 - c) : c);
  return slot < nunits ? (nunits - 1 - slot) : -1;
}

template <int CAP>
struct TopList {
  float sc[CAP];
  int ix[CAP];
  int n;
  float thr;  // score of the last entry when full

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int i = 0; i < CAP; ++i) { sc[i] = -INFINITY; ix[i] = 0x7fffffff; }
    n = 0;
    thr = -INFINITY;
  }
  // Candidates arrive with ascending j; a full list only takes a strictly
  // higher score than its last entry.
  __device__ __forceinline__ void offer(float s, int j, int cap) {
    if (cap == CAP && n == CAP) {
      offer_full(s, j);
      return;
    }
    if (n >= cap && !(s > thr)) return;
    bool gt[CAP];
#pragma unroll
    for (int i = 0; i < CAP; ++i) gt[i] = (i >= n) || (s > sc[i]);
#pragma unroll
    for (int i = CAP - 1; i >= 1; --i) {
      if (i < cap) {
        const float ns = gt[i - 1] ? sc[i - 1] : (gt[i] ? s : sc[i]);
        const int ni = gt[i - 1] ? ix[i - 1] : (gt[i] ? j : ix[i]);
        sc[i] = ns;
        ix[i] = ni;
      }
    }
    if (gt[0]) { sc[0] = s; ix[0] = j; }
    n = min(n + 1, cap);
    // the list is sorted descending, so its minimum is the last entry (a min
    // reduction keeps the list in registers; a select on cap-1 would not)
    float t = INFINITY;
#pragma unroll
    for (int i = 0; i < CAP; ++i) t = fminf(t, (i < cap) ? sc[i] : INFINITY);
    thr = t;
  }
  // The common case: all CAP entries in use (cap == CAP).  Sorted descending,
  // so the threshold is the last entry; no capacity checks, no min pass.
  __device__ __forceinline__ void offer_full(float s, int j) {
    if (!(s > sc[CAP - 1])) return;
    bool gt[CAP];
#pragma unroll
    for (int i = 0; i < CAP; ++i) gt[i] = s > sc[i];
#pragma unroll
    for (int i = CAP - 1; i >= 1; --i) {
      const float ns = gt[i - 1] ? sc[i - 1] : (gt[i] ? s : sc[i]);
      const int ni = gt[i - 1] ? ix[i - 1] : (gt[i] ? j : ix[i]);
      sc[i] = ns;
      ix[i] = ni;
    }
    if (gt[0]) { sc[0] = s; ix[0] = j; }
    thr = sc[CAP - 1];
  }
  // Write the selection ascending: the n chosen ids, then the local block,
  // then -1 padding.
  __device__ __forceinline__ void write(int32_t* dst, int k, int lb) const {
#pragma unroll
    for (int i = 0; i < CAP; ++i) {
      if (i < n) {
        int rank = 0;
#pragma unroll
        for (int j2 = 0; j2 < CAP; ++j2) rank += (j2 < n && ix[j2] < ix[i]) ? 1 : 0;
        dst[rank] = ix[i];
      }
    }
    dst[n] = lb;
    for (int r = n + 1; r < k; ++r) dst[r] = -1;
  }
};

// Max of 32 scores as a tree of 2-input fmaxf (ALU pipe; the 3-input form
// issues on the much narrower XU pipe).
__device__ __forceinline__ float max_of_32(const uint32_t (&r)[32]) {
  float m[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) m[i] = fmaxf(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) m[i] = fmaxf(m[i], m[i + w]);
  return m[0];
}

template <int KMAX, int G>
__global__ void __launch_bounds__(kThreads, 1)
index_topk_prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          int32_t* __restrict__ sel, const int32_t* __restrict__ cu_q,
                          const int32_t* __restrict__ cu_k, int batch, int d_idx, int k, int B_k, int nst,
                          int64_t row0, int64_t row1, DevError* err) {
  constexpr int CAP = KMAX - 1;
  constexpr int GP = G < 2 ? G : 2;          // groups per work unit
  constexpr int NPAIR = (G + GP - 1) / GP;   // units per tile
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);

  const int span = d_idx * 2 >= 128 ? 128 : d_idx * 2;   // bytes per swizzled row
  const int span_el = span / 2;
  const int nbox = (d_idx * 2) / span;                    // boxes per 128-row tile
  const uint32_t tile_bytes = kTile * d_idx * 2;          // one [128 x d_idx] bf16 tile
  uint8_t* q_s = smem;                                    // GP tiles
  uint8_t* k_s = smem + GP * tile_bytes;                  // nst tiles
  IndexCtl* ctl = reinterpret_cast<IndexCtl*>(k_s + nst * tile_bytes);
  volatile int32_t* abort_flag = &ctl->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&ctl->q_full, 1);
    mbar_init(&ctl->q_empty, GP);
    for (int s = 0; s < kStages; ++s) { mbar_init(&ctl->k_full[s], 1); mbar_init(&ctl->k_empty[s], GP); }
    for (int b = 0; b < 2; ++b)
      for (int l = 0; l < 2; ++l) { mbar_init(&ctl->acc_full[b][l], 1); mbar_init(&ctl->acc_empty[b][l], 4); }
    mbar_init(&ctl->mma_done[0], 1);
    mbar_init(&ctl->mma_done[1], 1);
    ctl->abort_flag = 0;
    // tiles per sequence (sequences with T_b > S_b are rejected and skipped)
    int acc = 0;
    for (int b = 0; b < batch; ++b) {
      ctl->tile_prefix[b] = acc;
      const int Tb = cu_q[b + 1] - cu_q[b];
      const int Sb = cu_k[b + 1] - cu_k[b];
      if (Tb < 0 || Tb > Sb) {
        report_error(err, MSA_ERR_DEVICE_CHECK, kSiteIndexSeq, b, Tb);
        continue;
      }
      acc += (Tb + kTile - 1) / kTile;
    }
    ctl->tile_prefix[batch] = acc;
    // this launch takes the tiles whose first row lies in [row0, row1) (first
    // rows grow with the tile index, so that is a contiguous range)
    auto first_at_or_after = [&](int64_t row) {
      int lo = 0, hi = acc;   // smallest tau with q0(tau) >= row
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        int b = 0, bh = batch;
        while (bh - b > 1) {
          const int m2 = (b + bh) >> 1;
          if (ctl->tile_prefix[m2] <= mid) b = m2; else bh = m2;
        }
        const int64_t q0 = (int64_t)cu_q[b] + (int64_t)kTile * (mid - ctl->tile_prefix[b]);
        if (q0 >= row) hi = mid; else lo = mid + 1;
      }
      return lo;
    };
    const int t0 = first_at_or_after(row0);
    const int t1 = first_at_or_after(row1);
    ctl->tau0 = t0;
    ctl->ntiles = t1 > t0 ? t1 - t0 : 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  const int nunits = ctl->ntiles * NPAIR;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      uint32_t kstep = 0, qiter = 0;
      for (int it = 0;; ++it) {
        const int u = snake_unit(it, nunits);
        if (u < 0 || *abort_flag) break;
        const int pair = u % NPAIR;
        const TileInfo ti = tile_info(ctl->tau0 + u / NPAIR, ctl, batch, cu_q, cu_k, B_k);
        if (!mbar_wait(&ctl->q_empty, (qiter + 1) & 1)) {
          report_error(err, MSA_ERR_TIMEOUT, kSiteIndexProducer, u, -1);
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&ctl->q_full, GP * tile_bytes);
        for (int l = 0; l < GP; ++l)
          for (int bx = 0; bx < nbox; ++bx)
            tma_load_3d(q_s + l * tile_bytes + bx * kTile * span, &tm_q, &ctl->q_full, bx * span_el,
                        pair * GP + l, ti.q0);
        ++qiter;
        for (int j = 0; j < ti.n_kb; ++j) {
          const int st = kstep % nst;
          if (!mbar_wait(&ctl->k_empty[st], ((kstep / nst) + 1) & 1)) {
            report_error(err, MSA_ERR_TIMEOUT, kSiteIndexProducer, u, j);
            *abort_flag = 1;
            break;
          }
          mbar_arrive_expect_tx(&ctl->k_full[st], tile_bytes);
          for (int bx = 0; bx < nbox; ++bx)
            tma_load_2d(k_s + st * tile_bytes + bx * kTile * span, &tm_k, &ctl->k_full[st], bx * span_el,
                        ti.k0row + kBk * j);
          ++kstep;
          if (*abort_flag) break;
        }
      }
      // Drain: every load this thread issued has landed before the CTA exits.
      if (qiter > 0) mbar_wait(&ctl->q_full, (qiter - 1) & 1);
      for (int st = 0; st < nst; ++st) {
        const uint32_t issued = kstep > (uint32_t)st ? (kstep - st + nst - 1) / nst : 0;
        if (issued > 0) mbar_wait(&ctl->k_full[st], (issued - 1) & 1);
      }
    }
  } else if (warp >= kMmaWarp && warp < kMmaWarp + GP) {
    if (lane == 0) {
      const int l = warp - kMmaWarp;   // group slot issued by this thread
      const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t mode = sw_mode_for(span);
      const uint32_t sbo = 8 * span;
      // descriptors are built once; each K=16 step adds its byte offset (>> 4)
      // to the start-address field
      const int nk = d_idx / 16;
      const int per_sh = span == 128 ? 2 : (span == 64 ? 1 : 0);   // log2(K steps per swizzled row)
      const uint64_t adesc = make_sdesc(smem_u32(q_s + l * tile_bytes), 16, sbo, mode);
      const uint64_t kdesc0 = make_sdesc(smem_u32(k_s), 16, sbo, mode);
      uint32_t kstep = 0, jstep = 0, qiter = 0;   // jstep: key blocks issued (all units)
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const int u = snake_unit(it, nunits);
        if (u < 0 || *abort_flag) break;
        const TileInfo ti = tile_info(ctl->tau0 + u / NPAIR, ctl, batch, cu_q, cu_k, B_k);
        if (!mbar_wait(&ctl->q_full, qiter & 1)) {
          report_error(err, MSA_ERR_TIMEOUT, kSiteIndexMma, u, -1);
          ok = false;
          break;
        }
        ++qiter;
        tc_fence_after();
        for (int j = 0; j < ti.n_kb && ok; ++j, ++jstep) {
          const int st = kstep % nst;
          const int buf = jstep & 1;
          if (!mbar_wait(&ctl->k_full[st], (kstep / nst) & 1) ||
              !mbar_wait(&ctl->acc_empty[buf][l], ((jstep >> 1) + 1) & 1)) {
            report_error(err, MSA_ERR_TIMEOUT, kSiteIndexMma, u, j);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bdesc = kdesc0 + (uint64_t)((st * tile_bytes) >> 4);
          const uint32_t acc = tmem_base + (buf * 2 + l) * 128;
          for (int kk = 0; kk < nk; ++kk) {
            const uint64_t off =
                (uint64_t)((((kk >> per_sh) * (kTile * span)) + ((kk & ((1 << per_sh) - 1)) * 32)) >> 4);
            umma_bf16_ss(acc, adesc + off, bdesc + off, idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(&ctl->acc_full[buf][l]);
          umma_commit(&ctl->k_empty[st]);
          ++kstep;
          if (*abort_flag) ok = false;
        }
        // the Q tile is reused only after every group's MMAs are done
        umma_commit(&ctl->q_empty);
      }
      if (!ok) *abort_flag = 1;
      // All issued MMAs complete before TMEM is released.
      umma_commit(&ctl->mma_done[l]);
      mbar_wait(&ctl->mma_done[l], 0);
    }
  } else if (warp < 4 * GP) {
    // ------------------------------------------------------------ epilogue
    const int l = warp / 4;            // group slot of this set within the unit
    const int wq = warp % 4;           // TMEM lane quarter
    const int row = 32 * wq + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(32 * wq) << 16) + l * 128;   // + buf * 256
    TopList<CAP> list;
    uint32_t jstep = 0;
    for (int it = 0;; ++it) {
      const int u = snake_unit(it, nunits);
      if (u < 0 || *abort_flag) break;
      const int g = (u % NPAIR) * GP + l;
      const TileInfo ti = tile_info(ctl->tau0 + u / NPAIR, ctl, batch, cu_q, cu_k, B_k);
      const bool valid = row < ti.rows;
      const int lb = (ti.pos0 + row) / B_k;
      list.reset();
      bool ok = true;
      for (int j = 0; j < ti.n_kb; ++j, ++jstep) {
        const int buf = jstep & 1;
        if (!mbar_wait(&ctl->acc_full[buf][l], (jstep >> 1) & 1)) {
          report_error(err, MSA_ERR_TIMEOUT, kSiteIndexEpilogue, u, j);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ta = lane_base + buf * 256;
        uint32_t r0[32], r1[32];
        tmem_ld32(ta, r0);
        tmem_ld32(ta + 32, r1);
        tmem_ld_wait();
        const float m0 = max_of_32(r0), m1 = max_of_32(r1);
        tmem_ld32(ta + 64, r0);
        tmem_ld32(ta + 96, r1);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->acc_empty[buf][l]);
        const float m2 = max_of_32(r0), m3 = max_of_32(r1);
        // the tile's 128 keys hold 128 / B_k blocks; offered in ascending order
        // (a block of NaN scores ranks as -inf)
        auto offer = [&](float m, int b) {
          if (m != m) m = -INFINITY;
          if (valid && b < lb) list.offer(m, b, k - 1);
        };
        if (B_k == kBk) {
          offer(fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)), j);
        } else if (B_k == 64) {
          offer(fmaxf(m0, m1), 2 * j);
          offer(fmaxf(m2, m3), 2 * j + 1);
        } else {
          offer(m0, 4 * j);
          offer(m1, 4 * j + 1);
          offer(m2, 4 * j + 2);
          offer(m3, 4 * j + 3);
        }
      }
      if (!ok) break;
      if (valid) list.write(sel + (static_cast<int64_t>(ti.q0 + row) * G + g) * k, k, lb);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace

int launch_index_topk_prefill(const IndexTopkArgs& a, void* stream) {
  const int span = a.d_idx * 2 >= 128 ? 128 : a.d_idx * 2;
  alignas(64) CUtensorMap tm_q, tm_k;
  {
    const uint64_t dims[3] = {(uint64_t)a.d_idx, (uint64_t)a.G, (uint64_t)a.total_q};
    const uint64_t strides[2] = {(uint64_t)a.d_idx * 2, (uint64_t)a.G * a.d_idx * 2};
    const uint32_t box[3] = {(uint32_t)(span / 2), 1u, (uint32_t)kTile};
    int rc = make_tmap_bf16(&tm_q, a.q_idx, 3, dims, strides, box, span);
    if (rc) return rc;
  }
  {
    const uint64_t dims[2] = {(uint64_t)a.d_idx, (uint64_t)a.total_k};
    const uint64_t strides[1] = {(uint64_t)a.d_idx * 2};
    const uint32_t box[2] = {(uint32_t)(span / 2), (uint32_t)kTile};
    int rc = make_tmap_bf16(&tm_k, a.k_idx, 2, dims, strides, box, span);
    if (rc) return rc;
  }
  const size_t tile_bytes = (size_t)kTile * a.d_idx * 2;
  const int gp = a.G < 2 ? a.G : 2;
  const int nst = a.d_idx >= 128 ? 4 : kStages;   // keep gp + nst tiles within shared memory
  size_t smem = 1024 + gp * tile_bytes + nst * tile_bytes + sizeof(IndexCtl);
  // at least 116 KB so that exactly one CTA (and one 512-column TMEM owner) sits on each SM
  if (smem < 116 * 1024) smem = 116 * 1024;
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int grid = a.grid > 0 && a.grid < nsm ? a.grid : nsm;
  const int64_t row1 = a.row1 > 0 ? a.row1 : a.total_q;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaErrorInvalidValue;
#define MSA_IDX(KM, GG)                                                                                        \
  if (a.k <= KM && a.G == GG) {                                                                                \
    e = cudaFuncSetAttribute(index_topk_prefill_kernel<KM, GG>, cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                             (int)smem);                                                                       \
    if (e != cudaSuccess) return (int)e;                                                                       \
    ProfScope p("index_topk_prefill", stream);                                                                 \
    index_topk_prefill_kernel<KM, GG><<<grid, kThreads, smem, st>>>(tm_q, tm_k, a.sel, a.cu_q, a.cu_k, a.batch, \
                                                                    a.d_idx, a.k, a.B_k, nst, a.row0, row1,   \
                                                                    a.err);                                   \
    return (int)cudaGetLastError();                                                                            \
  }
  MSA_IDX(8, 1) MSA_IDX(8, 2) MSA_IDX(8, 4)
  MSA_IDX(16, 1) MSA_IDX(16, 2) MSA_IDX(16, 4)
  MSA_IDX(32, 1) MSA_IDX(32, 2) MSA_IDX(32, 4)
#undef MSA_IDX
  return (int)e;
}

}  // namespace msa
