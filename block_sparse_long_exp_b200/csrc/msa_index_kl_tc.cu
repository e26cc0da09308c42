// msa_index_kl_tc.cu — the index-alignment target KL(P || Q) of every (query,
// group) on the tensor cores, for the selected support (pnsm.cn sec. 4 "KL
// alignment"; yhxrc.cn sec. 二; the quantities as msa_kl_unit.cuh defines
// them: teacher P_j = mean over the group's heads of exp(sm_scale q_h.k_j -
// lse_h), student Q_j = softmax_J(tau q_idx.k_idx_j)).
//
// The work is the forward's KV-outer work without its PV product: the
// selection is inverted into per-(group, window, block) query lists (the
// forward's planning, every selection on the lists), and each work item
// loads its key block and index-key rows once and gathers its queries' rows.
// kl_items_kernel (persistent, one CTA per SM, 384 threads):
//   warp 0      claims items (atomic ticket), publishes them in a ring and
//               loads each item's key block (TMA), its index-key rows (a bulk
//               copy that stops at the end of the keys) and, per 128-row
//               tile, the gathered query rows (one TMA box per query);
//   warp 1      owns TMEM (two S slots of 128 columns); lane 0 issues
//               S = Q K^T per tile (tile t in slot t % 2);
//   warps 4-11  two warpgroups, one per S slot: per row (query, head) P_h =
//               exp(sm_scale s - lse_h) for the block's keys in the support;
//               the mean over the query's head rows by warp shuffles; each
//               lane of a query then takes every RQ-th key: z = tau
//               q_idx.k_idx (CUDA cores, the index rows from shared memory)
//               and the KL's partial sums A = sum P log P, B = sum P z and a
//               (max, sum) pair of z; the lanes' partials are merged and
//               written as one float4 per (query, group, selected slot).
// kl_merge_kernel: per (query, group) the float4s of its slots give KL =
// sum A - sum B + log-sum-exp of z, and the student's log-sum-exp.
#include <cuda_runtime.h>

#include "msa_common.cuh"
#include "msa_internal.h"
#include "msa_kl.h"

namespace msa {
namespace {

constexpr int kKtThreads = 384;
constexpr int kKtItemRing = 4;
constexpr int kKtItemEmptyCount = 9;   // MMA issuer 1 + KL warps 8
constexpr int kKtKvEmptyCount = 9;     // the MMAs' commit + KL warps 8 (they read the index rows)
constexpr int kKtMaxQpw = 4;           // queries per warp (32 / RQ, RQ >= 8)

struct __align__(16) KtItem {
  int32_t seq, blk, g, start, count, Tb, Sb, qrow0;
};

struct __align__(16) KtCtl {
  uint64_t item_full[kKtItemRing], item_empty[kKtItemRing];
  uint64_t kv_full[2], kv_empty[2];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[2], s_free[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int32_t abort_flag;
  KtItem ring[kKtItemRing];
};

__global__ void __launch_bounds__(kKtThreads, 1)
kl_items_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                const uint16_t* __restrict__ k_idx, const uint16_t* __restrict__ q_idx,
                const float* __restrict__ lse, const Item* __restrict__ items, const int32_t* __restrict__ nitems_p,
                int32_t* __restrict__ ticket, const uint32_t* __restrict__ entries, const int32_t* __restrict__ cu_q,
                const int32_t* __restrict__ cu_k, int H, int G, int d, int d_idx, int k, float scale_log2,
                float temp, int64_t total_k, float4* __restrict__ part, DevError* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const int tile_bytes = 128 * d * 2;          // one [128 x d] bf16 tile
  const int kidx_bytes = 128 * d_idx * 2;      // one block of index-key rows
  uint8_t* k_s = smem;                          // 2 stages of K
  uint8_t* q_s = k_s + 2 * tile_bytes;          // 2 slots of gathered Q rows
  uint16_t* ki_s = reinterpret_cast<uint16_t*>(q_s + 2 * tile_bytes);            // 2 stages of index rows
  float* qi_s = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ki_s) + 2 * kidx_bytes);   // per KL warp
  float* pb_s = qi_s + 8 * kKtMaxQpw * d_idx;   // per KL warp and query: a chunk's 32 head-summed P
  KtCtl* ctl = reinterpret_cast<KtCtl*>(pb_s + 8 * kKtMaxQpw * 32);
  volatile int32_t* abort_flag = &ctl->abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hg = H / G;
  const int RQ = Hg < 8 ? 8 : Hg;               // tile rows per query
  const int qpt = 128 / RQ;                     // queries per 128-row tile
  const int nhalf = d / 64;
  const int nitems = *nitems_p;
  constexpr float kLog2e = 1.4426950408889634f;

  if (tid == 0) {
    for (int i = 0; i < kKtItemRing; ++i) {
      mbar_init(&ctl->item_full[i], 1);
      mbar_init(&ctl->item_empty[i], kKtItemEmptyCount);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->kv_full[i], 1);
      mbar_init(&ctl->kv_empty[i], kKtKvEmptyCount);
      mbar_init(&ctl->q_full[i], 1);
      mbar_init(&ctl->q_empty[i], 1);
      mbar_init(&ctl->s_full[i], 1);
      mbar_init(&ctl->s_free[i], 4);
    }
    mbar_init(&ctl->mma_done, 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_q);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;

  auto wait_item = [&](int n) -> const KtItem* {
    const int slot = n % kKtItemRing;
    if (!mbar_wait(&ctl->item_full[slot], (n / kKtItemRing) & 1)) {
      report_error(err, MSA_ERR_TIMEOUT, kSiteIndexKl, n, warp);
      *abort_flag = 1;
      return nullptr;
    }
    return &ctl->ring[slot];
  };

  if (warp == 0) {
    // ------------------------------------------ scheduler and every load
    int n = 0, tau = 0;
    bool ok = true;
    while (ok) {
      const int slot = n % kKtItemRing;
      if (lane == 0) ok = mbar_wait(&ctl->item_empty[slot], ((n / kKtItemRing) + 1) & 1);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      int it = 0;
      if (lane == 0) it = *abort_flag ? nitems : atomicAdd(ticket, 1);
      it = __shfl_sync(0xffffffffu, it, 0);
      KtItem* R = &ctl->ring[slot];
      if (it >= nitems) {
        if (lane == 0) {
          R->count = 0;
          mbar_arrive(&ctl->item_full[slot]);
        }
        break;
      }
      const Item I = items[it];
      const uint32_t e0 = lane < I.count ? entries[I.start + lane] : 0u;
      const uint32_t e1 = lane + 32 < I.count ? entries[I.start + lane + 32] : 0u;
      if (lane == 0) {
        R->seq = I.seq; R->blk = I.blk; R->g = I.g; R->start = I.start; R->count = I.count;
        R->Tb = cu_q[I.seq + 1] - cu_q[I.seq];
        R->Sb = cu_k[I.seq + 1] - cu_k[I.seq];
        R->qrow0 = cu_q[I.seq];
        mbar_arrive(&ctl->item_full[slot]);
        // the block's keys (TMA fills rows past the keys with zeros) and its
        // index rows (a plain bulk copy: it stops at the last key row)
        const int st = n & 1;
        ok = mbar_wait(&ctl->kv_empty[st], ((n >> 1) + 1) & 1);
        if (ok) {
          const int64_t krow = (int64_t)cu_k[I.seq] + (int64_t)I.blk * kBk;
          const int64_t rows = total_k - krow < kBk ? total_k - krow : kBk;
          const uint32_t ibytes = (uint32_t)(rows > 0 ? rows : 0) * (uint32_t)d_idx * 2u;
          mbar_arrive_expect_tx(&ctl->kv_full[st], (uint32_t)tile_bytes + ibytes);
          for (int h = 0; h < nhalf; ++h)
            tma_load_3d(k_s + st * tile_bytes + h * 128 * 128, &tm_k, &ctl->kv_full[st], 64 * h, I.g, (int)krow);
          if (ibytes > 0)
            bulk_load(reinterpret_cast<uint8_t*>(ki_s) + st * kidx_bytes, k_idx + krow * d_idx, ibytes,
                      &ctl->kv_full[st]);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      const int ntiles = (I.count + qpt - 1) / qpt;
      for (int mt = 0; ok && mt < ntiles; ++mt, ++tau) {
        const int qs = tau & 1;
        if (lane == 0) ok = mbar_wait(&ctl->q_empty[qs], ((tau >> 1) + 1) & 1);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        const int nq = min(qpt, I.count - mt * qpt);
        uint8_t* dst = q_s + qs * tile_bytes;
        if (lane == 0) mbar_arrive_expect_tx(&ctl->q_full[qs], nq * RQ * d * 2);
        __syncwarp();
        const int j = mt * qpt + lane;
        const uint32_t ej = __shfl_sync(0xffffffffu, e0, j & 31);
        const uint32_t ek = __shfl_sync(0xffffffffu, e1, j & 31);
        if (lane < nq) {
          const int64_t t = (j < 32 ? ej : ek) / k;   // the pass covers every query (t0 = 0)
          const int row = (int)(t * H + (int64_t)I.g * Hg);
          for (int h = 0; h < nhalf; ++h)
            tma_load_2d(dst + h * 128 * 128 + lane * RQ * 128, &tm_q, &ctl->q_full[qs], 64 * h, row);
        }
      }
      if (!ok) break;
      ++n;
    }
    if (lane == 0) {
      if (!ok) {
        report_error(err, MSA_ERR_TIMEOUT, kSiteIndexKl, n, -1);
        *abort_flag = 1;
      }
      // no load may still be in flight when the CTA exits
      for (int st = 0; st < 2; ++st) {
        const int issued = n > st ? (n - st + 1) / 2 : 0;
        if (issued > 0) mbar_wait(&ctl->kv_full[st], (issued - 1) & 1);
      }
      for (int qs = 0; qs < 2; ++qs) {
        const int issued = tau > qs ? (tau - qs + 1) / 2 : 0;
        if (issued > 0) mbar_wait(&ctl->q_full[qs], (issued - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      const uint64_t qdesc0 = make_sdesc(smem_u32(q_s), 16, 1024, kSw128);
      const uint64_t kdesc0 = make_sdesc(smem_u32(k_s), 16, 1024, kSw128);
      int n = 0, tau = 0;
      bool ok = true;
      while (ok && !*abort_flag) {
        const KtItem* R = wait_item(n);
        if (R == nullptr) { ok = false; break; }
        const int cnt = R->count;
        if (lane == 0) mbar_arrive(&ctl->item_empty[n % kKtItemRing]);
        if (cnt <= 0) break;
        const int st = n & 1;
        const int ntiles = (cnt + qpt - 1) / qpt;
        for (int mt = 0; mt < ntiles && ok; ++mt, ++tau) {
          const int s = tau & 1;
          if (!mbar_wait(&ctl->q_full[s], (tau >> 1) & 1) ||
              (mt == 0 && !mbar_wait(&ctl->kv_full[st], (n >> 1) & 1)) ||
              !mbar_wait(&ctl->s_free[s], ((tau >> 1) + 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t qd = qdesc0 + (uint64_t)((s * tile_bytes) >> 4);
          const uint64_t kd = kdesc0 + (uint64_t)((st * tile_bytes) >> 4);
          for (int kk = 0; kk < d / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4);
            umma_bf16_ss(tmem + s * 128, qd + off, kd + off, idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(&ctl->s_full[s]);
          umma_commit(&ctl->q_empty[s]);
          if (mt == ntiles - 1) umma_commit(&ctl->kv_empty[st]);   // the item's S products read K
        }
        ++n;
      }
      if (!ok) {
        report_error(err, MSA_ERR_TIMEOUT, kSiteIndexKl, tau, -2);
        *abort_flag = 1;
      }
      umma_commit(&ctl->mma_done);
      mbar_wait(&ctl->mma_done, 0);
    }
  } else if (warp >= 4) {
    // -------------------------------------------------- KL rows and sums
    const int wg = (warp - 4) >> 2;           // S slot of this warpgroup
    const int wq = warp & 3;                  // TMEM lane quarter
    const int r = 32 * wq + lane;             // tile row
    const uint32_t s_col = tmem + wg * 128 + (static_cast<uint32_t>(32 * wq) << 16);
    const int ql = r / RQ, hi = r - ql * RQ;
    const int qw = (lane / RQ);               // this lane's query within the warp
    float* qrow = qi_s + ((warp - 4) * kKtMaxQpw + qw) * d_idx;   // its index query, as floats
    float* psum = pb_s + ((warp - 4) * kKtMaxQpw + qw) * 32;      // its chunk of head-summed P
    const float inv_hg = 1.f / (float)Hg;
    int n = 0, tau = 0;
    while (!*abort_flag) {
      const KtItem* R = wait_item(n);
      if (R == nullptr) break;
      const int count = R->count;
      if (count <= 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->item_empty[n % kKtItemRing]);
        break;
      }
      const int st = n & 1;
      const int Tb = R->Tb, Sb = R->Sb, g = R->g;
      const int64_t qrow0 = R->qrow0;
      const int64_t blk_first = (int64_t)R->blk * kBk;
      const uint16_t* kis = ki_s + st * 128 * d_idx;
      const int ntiles = (count + qpt - 1) / qpt;
      bool failed = false;
      for (int mt = 0; mt < ntiles && !failed; ++mt, ++tau) {
        if ((tau & 1) != wg) continue;
        const int idx = mt * qpt + ql;
        const bool qvalid = ql < qpt && idx < count;    // this row's query exists
        const bool valid = qvalid && hi < Hg;           // and its head
        const uint32_t e = qvalid ? entries[R->start + idx] : 0u;
        const int64_t t = e / k;
        int limit = -1;                                  // last key of the block in the support
        if (qvalid) {
          const int64_t lim = (int64_t)Sb - Tb + (t - qrow0) - blk_first;
          limit = lim >= kBk - 1 ? kBk - 1 : (int)lim;
        }
        const float lse2 = valid ? lse[t * H + (int64_t)g * Hg + hi] * kLog2e : 0.f;
        // this query's index row, staged as floats by its lanes
        __syncwarp();
        if (qvalid)
          for (int c = hi; c < d_idx; c += RQ) qrow[c] = __uint_as_float((uint32_t)q_idx[(t * G + g) * d_idx + c] << 16);
        __syncwarp();
        // the block's index rows must have landed (the S MMA waited for the same barrier phase)
        if (!mbar_wait(&ctl->s_full[wg], (uint32_t)((tau >> 1) & 1)) ||
            !mbar_wait(&ctl->kv_full[st], (uint32_t)((n >> 1) & 1))) {
          report_error(err, MSA_ERR_TIMEOUT, kSiteIndexKl, tau, 1);
          *abort_flag = 1;
          failed = true;
          break;
        }
        tc_fence_after();
        float A = 0.f, B = 0.f, m = -INFINITY, l = 0.f;
        uint32_t rr[32];
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
          tmem_ld32(s_col + 32 * c4, rr);
          tmem_ld_wait();
          // P of every head row, summed over the query's RQ rows (all lanes take part)
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int col = 32 * c4 + j;
            float p = (valid && col <= limit) ? ex2_approx(fmaf(__uint_as_float(rr[j]), scale_log2, -lse2)) : 0.f;
            for (int off = RQ >> 1; off > 0; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
            if (hi == 0) psum[j] = p;
          }
          __syncwarp();
          // lane hi of the query takes the chunk's keys j = hi (mod RQ); the index
          // dot product starts at a lane-dependent 8-element piece (the rows are
          // 16-byte aligned, so lanes reading different rows avoid the same banks)
          for (int j = hi; j < 32; j += RQ) {
            const int col = 32 * c4 + j;
            if (!(qvalid && col <= limit)) continue;
            const float pbar = psum[j] * inv_hg;
            const uint16_t* kr = kis + col * d_idx;
            const int npc = d_idx / 8;
            float zs = 0.f;
            for (int i8 = 0; i8 < npc; ++i8) {
              const int c0 = ((i8 + hi) % npc) * 8;
              const uint4 w = *reinterpret_cast<const uint4*>(kr + c0);
              const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int q2 = 0; q2 < 4; ++q2) {
                zs += qrow[c0 + 2 * q2] * __uint_as_float(wv[q2] << 16);
                zs += qrow[c0 + 2 * q2 + 1] * __uint_as_float(wv[q2] & 0xffff0000u);
              }
            }
            const float z = temp * zs;   // temp: the student's temperature tau
            if (pbar > 0.f) A += pbar * __logf(pbar);
            B += pbar * z;
            if (z > m) {
              l = l * __expf(m - z) + 1.f;
              m = z;
            } else {
              l += __expf(z - m);
            }
          }
          __syncwarp();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->s_free[wg]);
        // merge the RQ lanes of each query
        for (int off = RQ >> 1; off > 0; off >>= 1) {
          A += __shfl_xor_sync(0xffffffffu, A, off);
          B += __shfl_xor_sync(0xffffffffu, B, off);
          const float m2 = __shfl_xor_sync(0xffffffffu, m, off);
          const float l2 = __shfl_xor_sync(0xffffffffu, l, off);
          const float mm = fmaxf(m, m2);
          l = (l > 0.f ? l * __expf(m - mm) : 0.f) + (l2 > 0.f ? l2 * __expf(m2 - mm) : 0.f);
          m = mm;
        }
        if (qvalid && hi == 0) part[((int64_t)t * G + g) * k + (e % k)] = make_float4(A, B, m, l);
        __syncwarp();
      }
      // the item's index rows are read: its stage may be reused
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&ctl->kv_empty[st]);
        mbar_arrive(&ctl->item_empty[n % kKtItemRing]);
      }
      if (failed) break;
      ++n;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// KL and the student's log-sum-exp per (query, group) from the slots' partials
// (a slot without one holds zeros: l = 0).
__global__ void kl_merge_kernel(const float4* __restrict__ part, int64_t npairs, int k, float* __restrict__ kl,
                                float* __restrict__ lse_z) {
  const int64_t pr = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (pr >= npairs) return;
  float A = 0.f, B = 0.f, m = -INFINITY;
  for (int s = 0; s < k; ++s) {
    const float4 v = part[pr * k + s];
    if (v.w > 0.f) {
      A += v.x;
      B += v.y;
      m = fmaxf(m, v.z);
    }
  }
  float l = 0.f;
  for (int s = 0; s < k; ++s) {
    const float4 v = part[pr * k + s];
    if (v.w > 0.f) l += v.w * __expf(v.z - m);
  }
  kl[pr] = l > 0.f ? A - B + m + __logf(l) : 0.f;
  if (lse_z != nullptr) lse_z[pr] = l > 0.f ? m + __logf(l) : -INFINITY;
}

}  // namespace

size_t kl_tc_smem_bytes(int d, int d_idx) {
  return 1024 + 4 * (size_t)128 * d * 2 + 2 * (size_t)128 * d_idx * 2 + sizeof(float) * 8 * kKtMaxQpw * d_idx +
         sizeof(float) * 8 * kKtMaxQpw * 32 + sizeof(KtCtl);
}

int launch_index_kl_tc(const IndexKlArgs& a, const AttnArgs& plan, float4* part, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t npairs = a.total_q * a.G;
  if (npairs <= 0) return 0;
  cudaError_t e = cudaMemsetAsync(part, 0, sizeof(float4) * (size_t)npairs * a.k, st);
  if (e != cudaSuccess) return (int)e;
  int rc = launch_kv_plan(plan, stream);
  if (rc) return rc;
  alignas(64) CUtensorMap tm_k, tm_q;
  {
    const uint64_t dims[3] = {(uint64_t)a.d, (uint64_t)a.G, (uint64_t)plan.total_k};
    const uint64_t strides[2] = {(uint64_t)a.d * 2, (uint64_t)a.G * a.d * 2};
    const uint32_t box[3] = {64u, 1u, 128u};
    rc = make_tmap_bf16(&tm_k, a.key, 3, dims, strides, box, 128);
    if (rc) return rc;
  }
  {
    const int hg = a.H / a.G;
    const uint64_t dims[2] = {(uint64_t)a.d, (uint64_t)a.total_q * a.H};
    const uint64_t strides[1] = {(uint64_t)a.d * 2};
    const uint32_t box[2] = {64u, (uint32_t)(hg < 8 ? 8 : hg)};
    rc = make_tmap_bf16(&tm_q, a.q, 2, dims, strides, box, 128);
    if (rc) return rc;
  }
  const size_t smem = kl_tc_smem_bytes(a.d, a.d_idx);
  e = cudaFuncSetAttribute(kl_items_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  {
    ProfScope p("index_kl", stream);
    kl_items_kernel<<<nsm, kKtThreads, smem, st>>>(
        tm_k, tm_q, static_cast<const uint16_t*>(a.k_idx), static_cast<const uint16_t*>(a.q_idx), a.lse, plan.items,
        plan.nitems, plan.nitems + 1, plan.entries, a.cu_q, a.cu_k, a.H, a.G, a.d, a.d_idx, a.k,
        a.sm_scale * 1.4426950408889634f, a.tau, plan.total_k, part, a.err);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  {
    ProfScope p("index_kl_merge", stream);
    kl_merge_kernel<<<(unsigned)((npairs + 255) / 256), 256, 0, st>>>(part, npairs, a.k, a.kl, a.lse_z);
  }
  return (int)cudaGetLastError();
}

}  // namespace msa
