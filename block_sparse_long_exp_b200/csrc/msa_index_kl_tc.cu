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
//               loads each item's key block and index-key block (TMA) and,
//               per 128-row tile, the gathered query rows (one TMA box per
//               query);
//   warps 2, 3  per tile (alternating), the index-query operand: every row
//               (query, head) of the tile holds its query's index vector, so
//               Z = that operand times the index keys gives each row its
//               query's raw index scores;
//   warp 1      owns TMEM (two slots of 256 columns); lane 0 issues
//               S = Q K^T and Z = Q_idx K_idx^T per tile (tile t in slot t % 2);
//   warps 4-11  two warpgroups, one per slot: per row (query, head) P_h =
//               exp(sm_scale s - lse_h) for the block's keys in the support;
//               the head sum by a reduce-scatter over the query's RQ lanes
//               (each lane ends with the sums of 32 / RQ keys of every
//               32-key chunk and picks the same keys' z from its Z row), then
//               the KL's partial sums A = sum P log P, B = sum P z and a
//               (max, sum) pair of z; the lanes' partials are merged and
//               written as one float4 per (query, group, selected slot).
// kl_merge_kernel: per (query, group) the float4s of its slots give KL =
// sum A - sum B + log-sum-exp of z, and the student's log-sum-exp.
//
// The same kernel in its gradient form (GRAD) computes, from the same P-bar
// and z and the student's log-sum-exp of the forward, w_j = tau (Q_j - P-bar_j)
// per (query, key) of the tile (the derivative of the KL with respect to the
// raw index score, the teacher held constant) into a shared table; then each
// warpgroup adds dq_idx[t, g] += sum_j w_j k_idx[j] (a thread per (query,
// 8-column chunk), the keys split across threads where there are fewer than
// 128 such pairs) and dk_idx[j] += sum_t w_j q_idx[t, g] (a thread per key),
// both with vector reductions to global memory.
#include <cuda_runtime.h>

#include "msa_common.cuh"
#include "msa_internal.h"
#include "msa_kl.h"

namespace msa {
namespace {

constexpr int kKtThreads = 384;
constexpr int kKtItemRing = 4;
constexpr int kKtItemEmptyCount = 11;  // MMA issuer 1 + index-query warps 2 + KL warps 8
constexpr uint32_t kKtTmemCols = 512;  // per slot: S in columns [0, 128), Z in [128, 256)
constexpr size_t kKtSmemLimit = 232448;
constexpr int kWtStride = 132;         // floats per row of the gradient's w table (16-byte rows, banks offset by 4)

struct __align__(16) KtItem {
  int32_t seq, blk, g, start, count, Tb, Sb, qrow0;
  int32_t krow, pad0, pad1, pad2;
};

struct __align__(16) KtCtl {
  uint64_t item_full[kKtItemRing], item_empty[kKtItemRing];
  uint64_t kv_full[2], kv_empty[2];
  uint64_t q_full[2], qi_full[2], q_empty[2];
  uint64_t s_full[2], s_free[2];
  uint64_t w_ready[2], rd_done[2];      // gradient: per warpgroup, its w table written / read
  uint64_t mma_done;
  uint32_t tmem_base;
  int32_t abort_flag;
  KtItem ring[kKtItemRing];
};

// Sum of p over the RQ lanes of a query (RQ aligned lanes), scattered: a step
// at lane offset `off` halves the values a lane keeps (the upper half where
// its lane bit `off` is set) and adds the partner's copy of them.  After
// log2(RQ) steps lane hi holds the sums of keys [hi * W, hi * W + W), W = 32 /
// RQ, in p[0, W).  z is the same for every lane of the query; it follows the
// same selection, so z[i] is the value of the key of p[i].
template <int RQ>
__device__ __forceinline__ void head_reduce_scatter(float (&p)[32], float (&z)[32], int hi) {
#pragma unroll
  for (int off = RQ / 2, half = 16; off >= 1; off >>= 1, half >>= 1) {
    const bool up = (hi & off) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = up ? p[i] : p[i + half];
      const float keep = up ? p[i + half] : p[i];
      p[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
      z[i] = up ? z[i + half] : z[i];
    }
  }
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ void red_add4(float* dst, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

// Shared bytes of the gradient's tables: per warpgroup a w table [qpt x 128]
// (rows of kWtStride floats) and the tile's index queries as floats [qpt x d_idx].
__host__ __device__ constexpr size_t kl_grad_bytes(int qpt, int d_idx) {
  return 2 * (size_t)qpt * kWtStride * 4 + 2 * (size_t)qpt * d_idx * 4;
}

template <int RQ, bool GRAD>
__global__ void __launch_bounds__(kKtThreads, 1)
kl_items_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                const __grid_constant__ CUtensorMap tm_ki, const uint16_t* __restrict__ q_idx,
                const float* __restrict__ lse, const Item* __restrict__ items, const int32_t* __restrict__ nitems_p,
                int32_t* __restrict__ ticket, const uint32_t* __restrict__ entries, const int32_t* __restrict__ cu_q,
                const int32_t* __restrict__ cu_k, int H, int G, int d, int d_idx, int k, int nst, float scale_log2,
                float temp, float4* __restrict__ part, const float* __restrict__ lse_z, float* __restrict__ dq_idx,
                float* __restrict__ dk_idx, DevError* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const int tile_bytes = 128 * d * 2;          // one [128 x d] bf16 tile
  const int itile_bytes = 128 * d_idx * 2;     // one [128 x d_idx] bf16 tile
  const int span = d_idx * 2 >= 128 ? 128 : d_idx * 2;   // bytes per swizzled row of an index tile
  const int span_el = span / 2;
  const int nibox = (d_idx * 2) / span;        // boxes per index tile
  uint8_t* k_s = smem;                          // nst stages of K
  uint8_t* ki_s = k_s + nst * tile_bytes;       // nst stages of K_idx
  uint8_t* q_s = ki_s + nst * itile_bytes;      // 2 slots of gathered Q rows
  uint8_t* qi_s = q_s + 2 * tile_bytes;         // 2 slots of the index-query operand
  constexpr int qpt = 128 / RQ;                 // queries per 128-row tile
  float* wt = reinterpret_cast<float*>(qi_s + 2 * itile_bytes);   // gradient tables (GRAD)
  float* qf = wt + 2 * qpt * kWtStride;
  KtCtl* ctl = reinterpret_cast<KtCtl*>(qi_s + 2 * itile_bytes + (GRAD ? kl_grad_bytes(qpt, d_idx) : 0));
  volatile int32_t* abort_flag = &ctl->abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hg = H / G;
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
      mbar_init(&ctl->kv_empty[i], GRAD ? 9 : 1);   // gradient: the KL warps read the index keys too
      mbar_init(&ctl->q_full[i], 1);
      mbar_init(&ctl->qi_full[i], 1);
      mbar_init(&ctl->q_empty[i], 1);
      mbar_init(&ctl->s_full[i], 1);
      mbar_init(&ctl->s_free[i], 4);
      mbar_init(&ctl->w_ready[i], 4);
      mbar_init(&ctl->rd_done[i], 4);
    }
    mbar_init(&ctl->mma_done, 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_ki);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, kKtTmemCols);
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
        const int krow = cu_k[I.seq] + I.blk * kBk;
        R->krow = krow;
        mbar_arrive(&ctl->item_full[slot]);
        // the block's keys and index keys (TMA fills rows past the keys with zeros)
        const int st = n % nst;
        ok = mbar_wait(&ctl->kv_empty[st], ((n / nst) + 1) & 1);
        if (ok) {
          mbar_arrive_expect_tx(&ctl->kv_full[st], (uint32_t)(tile_bytes + itile_bytes));
          for (int h = 0; h < nhalf; ++h)
            tma_load_3d(k_s + st * tile_bytes + h * 128 * 128, &tm_k, &ctl->kv_full[st], 64 * h, I.g, krow);
          for (int bx = 0; bx < nibox; ++bx)
            tma_load_2d(ki_s + st * itile_bytes + bx * 128 * span, &tm_ki, &ctl->kv_full[st], bx * span_el, krow);
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
      for (int st = 0; st < nst; ++st) {
        const int issued = n > st ? (n - st + nst - 1) / nst : 0;
        if (issued > 0) mbar_wait(&ctl->kv_full[st], (issued - 1) & 1);
      }
      for (int qs = 0; qs < 2; ++qs) {
        const int issued = tau > qs ? (tau - qs + 1) / 2 : 0;
        if (issued > 0) mbar_wait(&ctl->q_full[qs], (issued - 1) & 1);
      }
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------- index-query operand of every other tile
    // row r of the tile holds q_idx[t, g] of its query r / RQ, in the
    // swizzled K-major layout the index keys' TMA writes
    const int my = warp - 2;
    const int cpr = d_idx / 8;                 // 16-byte chunks per row
    const int cpb = span / 16;                 // chunks per box row
    const int nload = (qpt * cpr) / 32;        // chunks per lane (1 to 8)
    int n = 0, tau = 0;
    bool ok = true;
    while (ok && !*abort_flag) {
      const KtItem* R = wait_item(n);
      if (R == nullptr) break;
      const int count = R->count, start = R->start, g = R->g;
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->item_empty[n % kKtItemRing]);
      if (count <= 0) break;
      const int ntiles = (count + qpt - 1) / qpt;
      for (int mt = 0; mt < ntiles; ++mt, ++tau) {
        const int qs = tau & 1;
        if (qs != my) continue;
        if (lane == 0) ok = mbar_wait(&ctl->q_empty[qs], ((tau >> 1) + 1) & 1);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        const int nq = min(qpt, count - mt * qpt);
        const uint32_t e = lane < nq ? entries[start + mt * qpt + lane] : 0u;
        uint4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int u = lane + 32 * i, ql = u / cpr, c = u - ql * cpr;
          const uint32_t eq = __shfl_sync(0xffffffffu, e, ql & 31);
          v[i] = make_uint4(0u, 0u, 0u, 0u);
          if (i < nload && ql < nq)
            v[i] = *reinterpret_cast<const uint4*>(q_idx + ((int64_t)(eq / k) * G + g) * d_idx + c * 8);
        }
        uint8_t* dst = qi_s + qs * itile_bytes;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (i < nload) {
            const int u = lane + 32 * i, ql = u / cpr, c = u - ql * cpr;
            const int bx = c / cpb, cc = c - bx * cpb;
#pragma unroll
            for (int h = 0; h < RQ; ++h)
              *reinterpret_cast<uint4*>(dst + bx * 128 * span + swz_offset(ql * RQ + h, cc, span)) = v[i];
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->qi_full[qs]);
      }
      if (!ok) break;
      ++n;
    }
    if (!ok && lane == 0) {
      report_error(err, MSA_ERR_TIMEOUT, kSiteIndexKl, tau, -3);
      *abort_flag = 1;
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
      const uint64_t qdesc0 = make_sdesc(smem_u32(q_s), 16, 1024, kSw128);
      const uint64_t kdesc0 = make_sdesc(smem_u32(k_s), 16, 1024, kSw128);
      const uint32_t imode = sw_mode_for(span);
      const uint64_t qidesc0 = make_sdesc(smem_u32(qi_s), 16, 8 * span, imode);
      const uint64_t kidesc0 = make_sdesc(smem_u32(ki_s), 16, 8 * span, imode);
      const int per_sh = span == 128 ? 2 : (span == 64 ? 1 : 0);   // log2(K steps per swizzled row)
      int n = 0, tau = 0;
      bool ok = true;
      while (ok && !*abort_flag) {
        const KtItem* R = wait_item(n);
        if (R == nullptr) { ok = false; break; }
        const int cnt = R->count;
        mbar_arrive(&ctl->item_empty[n % kKtItemRing]);
        if (cnt <= 0) break;
        const int st = n % nst;
        const int ntiles = (cnt + qpt - 1) / qpt;
        for (int mt = 0; mt < ntiles && ok; ++mt, ++tau) {
          const int s = tau & 1;
          if (!mbar_wait(&ctl->q_full[s], (tau >> 1) & 1) || !mbar_wait(&ctl->qi_full[s], (tau >> 1) & 1) ||
              (mt == 0 && !mbar_wait(&ctl->kv_full[st], (n / nst) & 1)) ||
              !mbar_wait(&ctl->s_free[s], ((tau >> 1) + 1) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t qd = qdesc0 + (uint64_t)((s * tile_bytes) >> 4);
          const uint64_t kd = kdesc0 + (uint64_t)((st * tile_bytes) >> 4);
          for (int kk = 0; kk < d / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4);
            umma_bf16_ss(tmem + s * 256, qd + off, kd + off, idesc, kk > 0 ? 1u : 0u);
          }
          const uint64_t qid = qidesc0 + (uint64_t)((s * itile_bytes) >> 4);
          const uint64_t kid = kidesc0 + (uint64_t)((st * itile_bytes) >> 4);
          for (int kk = 0; kk < d_idx / 16; ++kk) {
            const uint64_t off =
                (uint64_t)((((kk >> per_sh) * (128 * span)) + ((kk & ((1 << per_sh) - 1)) * 32)) >> 4);
            umma_bf16_ss(tmem + s * 256 + 128, qid + off, kid + off, idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(&ctl->s_full[s]);
          umma_commit(&ctl->q_empty[s]);
          if (mt == ntiles - 1) umma_commit(&ctl->kv_empty[st]);   // the item's products read its key stage
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
    constexpr int W = 32 / RQ;                // keys per 32-key chunk a lane ends with
    const int wg = (warp - 4) >> 2;           // slot of this warpgroup
    const int wq = warp & 3;                  // TMEM lane quarter
    const int r = 32 * wq + lane;             // tile row
    const uint32_t s_col = tmem + wg * 256 + (static_cast<uint32_t>(32 * wq) << 16);
    const int ql = r / RQ, hi = r - ql * RQ;
    const float inv_hg = 1.f / (float)Hg;
    const int tw = 32 * wq + lane;            // thread of the warpgroup
    const int cpr8 = d_idx / 8;               // 8-column chunks per index row
    float* wt_g = wt + wg * qpt * kWtStride;  // gradient: this warpgroup's w table
    float* qf_g = qf + wg * qpt * d_idx;      // and its tile's index queries as floats
    int ktile = 0;                            // tiles this warpgroup has taken
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
      const int Tb = R->Tb, Sb = R->Sb, g = R->g, start = R->start;
      const int64_t krow = R->krow;
      const int st = n % nst;
      const int64_t qrow0 = R->qrow0;
      const int64_t blk_first = (int64_t)R->blk * kBk;
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->item_empty[n % kKtItemRing]);
      const int ntiles = (count + qpt - 1) / qpt;
      bool failed = false;
      for (int mt = 0; mt < ntiles; ++mt, ++tau) {
        if ((tau & 1) != wg) continue;
        const int idx = mt * qpt + ql;
        const bool qvalid = idx < count;                 // this row's query exists
        const bool valid = qvalid && hi < Hg;           // and its head
        const uint32_t e = qvalid ? entries[start + idx] : 0u;
        const int64_t t = e / k;
        int limit = -1;                                  // last key of the block in the support
        if (qvalid) {
          const int64_t lim = (int64_t)Sb - Tb + (t - qrow0) - blk_first;
          limit = lim >= kBk - 1 ? kBk - 1 : (int)lim;
        }
        const float lse2 = valid ? lse[t * H + (int64_t)g * Hg + hi] * kLog2e : 0.f;
        float lsez2 = 0.f;
        if constexpr (GRAD) {
          lsez2 = qvalid ? lse_z[t * G + g] * kLog2e : 0.f;
          // the previous tile's tables are read; this tile's index queries as floats
          if (ktile > 0 && !mbar_wait(&ctl->rd_done[wg], (uint32_t)((ktile - 1) & 1))) {
            report_error(err, MSA_ERR_TIMEOUT, kSiteIndexKl, tau, 2);
            *abort_flag = 1;
            failed = true;
            break;
          }
          for (int u2 = tw; u2 < qpt * cpr8; u2 += 128) {
            const int q2 = u2 / cpr8, c8 = u2 - q2 * cpr8;
            const int i2 = mt * qpt + q2;
            float4 lo = make_float4(0.f, 0.f, 0.f, 0.f), up = lo;
            if (i2 < count) {
              const int64_t t2 = entries[start + i2] / k;
              const uint4 v = *reinterpret_cast<const uint4*>(q_idx + (t2 * G + g) * d_idx + c8 * 8);
              lo = make_float4(bf_lo(v.x), bf_hi(v.x), bf_lo(v.y), bf_hi(v.y));
              up = make_float4(bf_lo(v.z), bf_hi(v.z), bf_lo(v.w), bf_hi(v.w));
            }
            *reinterpret_cast<float4*>(qf_g + q2 * d_idx + c8 * 8) = lo;
            *reinterpret_cast<float4*>(qf_g + q2 * d_idx + c8 * 8 + 4) = up;
          }
        }
        if (!mbar_wait(&ctl->s_full[wg], (uint32_t)((tau >> 1) & 1)) ||
            (GRAD && !mbar_wait(&ctl->kv_full[st], (uint32_t)((n / nst) & 1)))) {
          report_error(err, MSA_ERR_TIMEOUT, kSiteIndexKl, tau, 1);
          *abort_flag = 1;
          failed = true;
          break;
        }
        tc_fence_after();
        float A = 0.f, B = 0.f, m = -INFINITY, l = 0.f;
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t rs[32], rz[32];
          tmem_ld32(s_col + 32 * c4, rs);
          tmem_ld32(s_col + 128 + 32 * c4, rz);
          tmem_ld_wait();
          if (c4 == 3) {
            // the slot is read: the next tile's products may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->s_free[wg]);
          }
          float p[32], z[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int col = 32 * c4 + j;
            p[j] = (valid && col <= limit) ? ex2_approx(fmaf(__uint_as_float(rs[j]), scale_log2, -lse2)) : 0.f;
            z[j] = __uint_as_float(rz[j]);
          }
          head_reduce_scatter<RQ>(p, z, hi);
          if constexpr (GRAD) {
            // w = tau (Q - P-bar) of the lane's keys
#pragma unroll
            for (int i = 0; i < W; ++i) {
              const int col = 32 * c4 + W * hi + i;
              float w = 0.f;
              if (qvalid && col <= limit)
                w = temp * (ex2_approx(temp * z[i] * kLog2e - lsez2) - p[i] * inv_hg);
              wt_g[ql * kWtStride + col] = w;
            }
          } else {
#pragma unroll
            for (int i = 0; i < W; ++i) {
              const int col = 32 * c4 + W * hi + i;
              if (qvalid && col <= limit) {
                const float pbar = p[i] * inv_hg;
                const float zz = temp * z[i];
                if (pbar > 0.f) A += pbar * __logf(pbar);
                B += pbar * zz;
                if (zz > m) {
                  l = l * __expf(m - zz) + 1.f;
                  m = zz;
                } else {
                  l += __expf(zz - m);
                }
              }
            }
          }
        }
        if constexpr (GRAD) {
          // the tile's w table is complete once the warpgroup's four warps have written
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->w_ready[wg]);
          if (!mbar_wait(&ctl->w_ready[wg], (uint32_t)(ktile & 1))) {
            report_error(err, MSA_ERR_TIMEOUT, kSiteIndexKl, tau, 3);
            *abort_flag = 1;
            failed = true;
            break;
          }
          const int nq = min(qpt, count - mt * qpt);
          // dq_idx[t, g] += sum_j w_j k_idx[j]: a thread per (query, 8-column
          // chunk), the keys split over ks threads (adjacent lanes) where
          // there are fewer than 128 such pairs
          {
            const int pairs = qpt * cpr8;
            const int ks = pairs >= 128 ? 1 : 128 / pairs;
            const int per = pairs > 128 ? pairs / 128 : 1;
            const int nkeys = 128 / ks;
            const int split = tw % ks;
            const uint8_t* kst = ki_s + st * itile_bytes;
            for (int pp = 0; pp < per; ++pp) {
              const int pid = tw / ks + pp * (128 / ks);
              const int q2 = pid / cpr8, c8 = pid - q2 * cpr8;
              const int cel = c8 * 8, box = cel / span_el, cin = (cel - box * span_el) / 8;
              const uint8_t* kb = kst + box * 128 * span;
              const float* wr = wt_g + q2 * kWtStride;
              float acc[8];
#pragma unroll
              for (int e2 = 0; e2 < 8; ++e2) acc[e2] = 0.f;
              if (q2 < nq) {
#pragma unroll 4
                for (int jj = 0; jj < nkeys; ++jj) {
                  // each split starts at its own row (lanes reading the same chunk of rows
                  // 64 apart would meet in one bank)
                  const int j = split * nkeys + ((jj + split) & (nkeys - 1));
                  const float wv = wr[j];
                  const uint4 kv = *reinterpret_cast<const uint4*>(kb + swz_offset(j, cin, span));
                  acc[0] += wv * bf_lo(kv.x); acc[1] += wv * bf_hi(kv.x);
                  acc[2] += wv * bf_lo(kv.y); acc[3] += wv * bf_hi(kv.y);
                  acc[4] += wv * bf_lo(kv.z); acc[5] += wv * bf_hi(kv.z);
                  acc[6] += wv * bf_lo(kv.w); acc[7] += wv * bf_hi(kv.w);
                }
              }
              for (int off = 1; off < ks; off <<= 1) {
#pragma unroll
                for (int e2 = 0; e2 < 8; ++e2) acc[e2] += __shfl_xor_sync(0xffffffffu, acc[e2], off);
              }
              if (split == 0 && q2 < nq) {
                const int64_t t2 = entries[start + mt * qpt + q2] / k;
                float* dst = dq_idx + (t2 * G + g) * d_idx + cel;
                red_add4(dst, acc[0], acc[1], acc[2], acc[3]);
                red_add4(dst + 4, acc[4], acc[5], acc[6], acc[7]);
              }
            }
          }
          // dk_idx[j] += sum over the tile's queries of w_j q_idx[t, g]: a thread per key
          if (blk_first + tw < Sb) {
            float* dst = dk_idx + (krow + tw) * d_idx;
            for (int c0 = 0; c0 < d_idx; c0 += 32) {
              float acc[32];
#pragma unroll
              for (int e2 = 0; e2 < 32; ++e2) acc[e2] = 0.f;
              for (int q2 = 0; q2 < nq; ++q2) {
                const float wv = wt_g[q2 * kWtStride + tw];
                const float4* qr = reinterpret_cast<const float4*>(qf_g + q2 * d_idx + c0);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                  const float4 x = qr[c];
                  acc[4 * c] += wv * x.x; acc[4 * c + 1] += wv * x.y;
                  acc[4 * c + 2] += wv * x.z; acc[4 * c + 3] += wv * x.w;
                }
              }
#pragma unroll
              for (int c = 0; c < 8; ++c)
                red_add4(dst + c0 + 4 * c, acc[4 * c], acc[4 * c + 1], acc[4 * c + 2], acc[4 * c + 3]);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->rd_done[wg]);
          ++ktile;
        } else {
          // merge the RQ lanes of each query
#pragma unroll
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
        }
      }
      if (failed) break;
      if constexpr (GRAD) {
        // the item's index keys are read: its key stage may be reused.  A warp
        // whose warpgroup took none of the item's tiles first waits for the
        // item's keys to have landed: the item ring runs ahead of the key
        // stages, and without that wait such a warp could arrive for a later
        // item of the same stage before this item's phase completes.
        if (!mbar_wait(&ctl->kv_full[st], (uint32_t)((n / nst) & 1))) {
          report_error(err, MSA_ERR_TIMEOUT, kSiteIndexKl, n, 4);
          *abort_flag = 1;
          break;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->kv_empty[st]);
      }
      ++n;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kKtTmemCols);
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


// Key stages that fit beside the two query slots and, for the gradient, its
// tables (2 where the shared memory allows, else 1).
int kl_tc_stages(int d, int d_idx, size_t extra) {
  const size_t per = (size_t)128 * d * 2 + (size_t)128 * d_idx * 2;
  return 1024 + 4 * per + extra + sizeof(KtCtl) <= kKtSmemLimit ? 2 : 1;
}

size_t kl_tc_smem_bytes(int d, int d_idx, size_t extra) {
  const size_t per = (size_t)128 * d * 2 + (size_t)128 * d_idx * 2;
  return 1024 + (size_t)(kl_tc_stages(d, d_idx, extra) + 2) * per + extra + sizeof(KtCtl);
}

// Tensor maps of the key blocks (3D: column, group, row), the gathered query
// rows (one box per query: its group's head rows, at least 8) and the
// index-key blocks (swizzled as the index rows' width allows).
int kl_tc_maps(const IndexKlArgs& a, int64_t total_k, CUtensorMap* tm_k, CUtensorMap* tm_q, CUtensorMap* tm_ki) {
  {
    const uint64_t dims[3] = {(uint64_t)a.d, (uint64_t)a.G, (uint64_t)total_k};
    const uint64_t strides[2] = {(uint64_t)a.d * 2, (uint64_t)a.G * a.d * 2};
    const uint32_t box[3] = {64u, 1u, 128u};
    const int rc = make_tmap_bf16(tm_k, a.key, 3, dims, strides, box, 128);
    if (rc) return rc;
  }
  {
    const int hg = a.H / a.G;
    const uint64_t dims[2] = {(uint64_t)a.d, (uint64_t)a.total_q * a.H};
    const uint64_t strides[1] = {(uint64_t)a.d * 2};
    const uint32_t box[2] = {64u, (uint32_t)(hg < 8 ? 8 : hg)};
    const int rc = make_tmap_bf16(tm_q, a.q, 2, dims, strides, box, 128);
    if (rc) return rc;
  }
  const int span = a.d_idx * 2 >= 128 ? 128 : a.d_idx * 2;
  const uint64_t dims[2] = {(uint64_t)a.d_idx, (uint64_t)total_k};
  const uint64_t strides[1] = {(uint64_t)a.d_idx * 2};
  const uint32_t box[2] = {(uint32_t)(span / 2), 128u};
  return make_tmap_bf16(tm_ki, a.k_idx, 2, dims, strides, box, span);
}

// The persistent items kernel over the plan's lists: the target's partials
// (GRAD false) or the gradient's reductions into dq_idx / dk_idx.
template <bool GRAD>
int launch_items(const IndexKlArgs& a, const AttnArgs& plan, float4* part, const char* name, void* stream) {
  alignas(64) CUtensorMap tm_k, tm_q, tm_ki;
  int rc = kl_tc_maps(a, plan.total_k, &tm_k, &tm_q, &tm_ki);
  if (rc) return rc;
  const int hg = a.H / a.G;
  const int rq = hg <= 8 ? 8 : 16;
  const size_t extra = GRAD ? kl_grad_bytes(128 / rq, a.d_idx) : 0;
  const int nst = kl_tc_stages(a.d, a.d_idx, extra);
  const size_t smem = kl_tc_smem_bytes(a.d, a.d_idx, extra);
  auto kern = rq == 8 ? kl_items_kernel<8, GRAD> : kl_items_kernel<16, GRAD>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  {
    ProfScope p(name, stream);
    kern<<<nsm, kKtThreads, smem, reinterpret_cast<cudaStream_t>(stream)>>>(
        tm_k, tm_q, tm_ki, static_cast<const uint16_t*>(a.q_idx), a.lse, plan.items, plan.nitems,
        plan.nitems + 1, plan.entries, a.cu_q, a.cu_k, a.H, a.G, a.d, a.d_idx, a.k, nst,
        a.sm_scale * 1.4426950408889634f, a.tau, part, a.lse_z, a.dq_idx, a.dk_idx, a.err);
  }
  return (int)cudaGetLastError();
}

}  // namespace

int launch_index_kl_tc(const IndexKlArgs& a, const AttnArgs& plan, float4* part, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t npairs = a.total_q * a.G;
  if (npairs <= 0) return 0;
  cudaError_t e = cudaMemsetAsync(part, 0, sizeof(float4) * (size_t)npairs * a.k, st);
  if (e != cudaSuccess) return (int)e;
  int rc = launch_kv_plan(plan, stream);
  if (rc) return rc;
  rc = launch_items<false>(a, plan, part, "index_kl", stream);
  if (rc) return rc;
  {
    ProfScope p("index_kl_merge", stream);
    kl_merge_kernel<<<(unsigned)((npairs + 255) / 256), 256, 0, st>>>(part, npairs, a.k, a.kl, a.lse_z);
  }
  return (int)cudaGetLastError();
}

int launch_index_kl_grad_tc(const IndexKlArgs& a, const AttnArgs& plan, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t npairs = a.total_q * a.G;
  if (npairs <= 0) return 0;
  // both gradients are sums of the items' reductions
  cudaError_t e = cudaMemsetAsync(a.dq_idx, 0, sizeof(float) * (size_t)npairs * a.d_idx, st);
  if (e != cudaSuccess) return (int)e;
  int rc = launch_kv_plan(plan, stream);
  if (rc) return rc;
  return launch_items<true>(a, plan, nullptr, "index_kl_grad", stream);
}

}  // namespace msa
