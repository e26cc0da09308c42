// msa_attn_bwd_tc.cu — the Main Branch backward on the tensor cores, for the
// selected support (the forward that yifor-blog "設計核心" item 2 and pnsm.cn
// sec. 2 define, differentiated like any softmax attention: with P_j =
// exp(sm_scale q.k_j - lse), dP_j = dO.v_j, D = dO.O and dS_j = P_j (dP_j - D),
// dq = sm_scale sum_j dS_j k_j, dk_j += sm_scale dS_j q, dv_j += P_j dO).
//
// The work is the forward's KV-outer work: the selection is inverted into
// per-(group, window, block) query lists (the forward's planning), and each
// work item keeps its key and value block in shared memory while it walks its
// queries in tiles of 128 rows (query, head).  The products are taken with
// the keys on the TMEM lanes, so that P^T and dS^T stay in TMEM as the A
// operands of the dV and dK products:
//   S^T  = K Q^T,   dP^T = V dO^T               (SS, 128 x 128, K = d)
//   dV  += P^T dO,  dK  += dS^T Q                (TS, 128 x d, K = the tile's rows;
//                                                 dO and Q as MN-major B operands)
//   dQ   = dS K                                  (SS, 128 x d, K = the block's keys;
//                                                 dS written to shared memory, K MN-major)
// attn_bwd_items_kernel (persistent, one CTA per SM, 384 threads):
//   warp 0      claims items (atomic ticket), publishes them in a ring, loads
//               the item's K and V blocks (TMA) and each tile's gathered Q and
//               dO rows (one TMA box per query);
//   warp 1      owns TMEM (512 columns: S^T, dP^T, dV, dK) and issues the products;
//   warps 4-11  per tile: P^T and dS^T from S^T and dP^T (the rows' log-sum-
//               exps and D staged in shared memory), packed to bf16 into the
//               first halves of their own columns, and dS into shared memory;
//               warps 4-7 take the tile's rows 0..63, warps 8-11 rows 64..127;
//   warps 8-11  then, per tile: dQ (in the second halves of those columns)
//               added to dq with vector reductions; per item: dK and dV added
//               to dk and dv.
// The tile's steps run in order (TMEM holds one tile); the loads run ahead.
// rowdot_kernel: D[t, h] = dO[t, h] . O[t, h] (fp32), before the items.
#include <cuda_runtime.h>
#include <stddef.h>

#include "msa_bwd.h"
#include "msa_common.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kBtThreads = 384;
constexpr int kBtItemRing = 4;
constexpr int kBtItemEmptyCount = 9;   // MMA issuer 1 + P warps 4 + drain warps 4
constexpr uint32_t kBtTmemCols = 512;
constexpr size_t kBtSmemLimit = 232448;

struct __align__(16) BtItem {
  int32_t seq, blk, g, start, count, Tb, Sb, qrow0;
  int32_t krow, pad0, pad1, pad2;
};

struct __align__(16) BtCtl {
  uint64_t item_full[kBtItemRing], item_empty[kBtItemRing];
  uint64_t kv_full[2], kv_empty[2];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full, p_ready, dq_full, tmem_free, dkv_full, dkv_free, rows_ready[2], c1_read;
  uint64_t mma_done;
  uint32_t tmem_base;
  int32_t abort_flag;
  BtItem ring[kBtItemRing];
  // per tile row (two buffers by tile parity): log2-scaled log-sum-exp,
  // sm_scale * D, last visible key of the block (-1: no such row)
  float lse2[2][128];
  float dsc[2][128];
  int32_t lim[2][128];
};

static_assert(offsetof(BtCtl, lse2) % 16 == 0 && offsetof(BtCtl, dsc) % 16 == 0 && offsetof(BtCtl, lim) % 16 == 0,
              "the row tables are read 16 bytes at a time");

__device__ __forceinline__ void red_add4(float* dst, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

__device__ __forceinline__ int4 lds_i4(uint32_t addr) {
  int4 v;
  asm volatile("ld.shared.v4.s32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// D = dO . O per (query, head) row, one thread per row.
__global__ void rowdot_kernel(const uint16_t* __restrict__ dout, const uint16_t* __restrict__ out, int64_t rows,
                              int d, float* __restrict__ D) {
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  const uint4* a = reinterpret_cast<const uint4*>(dout + r * d);
  const uint4* b = reinterpret_cast<const uint4*>(out + r * d);
  float acc = 0.f;
  for (int c = 0; c < d / 8; ++c) {
    const uint4 x = a[c], y = b[c];
    const uint32_t xv[4] = {x.x, x.y, x.z, x.w}, yv[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc += __uint_as_float(xv[i] << 16) * __uint_as_float(yv[i] << 16);
      acc += __uint_as_float(xv[i] & 0xffff0000u) * __uint_as_float(yv[i] & 0xffff0000u);
    }
  }
  D[r] = acc;
}

template <int RQ>
__global__ void __launch_bounds__(kBtThreads, 1)
attn_bwd_items_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                      const uint16_t* __restrict__ qg, const uint16_t* __restrict__ dog,
                      const float* __restrict__ lse, const float* __restrict__ Dg, const Item* __restrict__ items,
                      const int32_t* __restrict__ nitems_p, int32_t* __restrict__ ticket,
                      const uint32_t* __restrict__ entries, const int32_t* __restrict__ cu_q,
                      const int32_t* __restrict__ cu_k, int H, int G, int d, int k, int nkv, int nq,
                      float scale_log2, float sm_scale, float* __restrict__ dq, float* __restrict__ dk,
                      float* __restrict__ dv, DevError* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const int tile_bytes = 128 * d * 2;          // one [128 x d] bf16 tile
  uint8_t* kv_s = smem;                         // nkv stages of [K | V]
  uint8_t* q_s = kv_s + nkv * 2 * tile_bytes;   // nq slots of [Q | dO]
  uint8_t* ds_s = q_s + nq * 2 * tile_bytes;    // dS [128 rows x 128 keys], K-major, 128-byte swizzle
  BtCtl* ctl = reinterpret_cast<BtCtl*>(ds_s + 128 * 128 * 2);
  volatile int32_t* abort_flag = &ctl->abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int Hg = H / G;
  constexpr int qpt = 128 / RQ;                 // queries per 128-row tile
  const int nhalf = d / 64;
  const int nitems = *nitems_p;

  if (tid == 0) {
    for (int i = 0; i < kBtItemRing; ++i) {
      mbar_init(&ctl->item_full[i], 1);
      mbar_init(&ctl->item_empty[i], kBtItemEmptyCount);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->kv_full[i], 1);
      mbar_init(&ctl->kv_empty[i], 1);
      mbar_init(&ctl->q_full[i], 1);
      mbar_init(&ctl->q_empty[i], 1);
    }
    mbar_init(&ctl->s_full, 1);
    mbar_init(&ctl->p_ready, 8);
    mbar_init(&ctl->dq_full, 1);
    mbar_init(&ctl->tmem_free, 4);
    mbar_init(&ctl->dkv_full, 1);
    mbar_init(&ctl->dkv_free, 4);
    mbar_init(&ctl->rows_ready[0], 4);
    mbar_init(&ctl->rows_ready[1], 4);
    mbar_init(&ctl->c1_read, 4);
    mbar_init(&ctl->mma_done, 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_do);
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, kBtTmemCols);
    tmem_relinquish();
  }
  // The Q / dO slots start as zeros: a tile's rows past its queries keep the
  // previous contents, which the dV and dK products multiply by zero, and
  // zero times a stale bf16 row is zero, whereas shared memory never written
  // may hold NaN patterns.
  for (int i = tid; i < nq * 2 * tile_bytes / 16; i += kBtThreads)
    reinterpret_cast<uint4*>(q_s)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  // TMEM columns: S^T [0, 128) (then P^T in [0, 64), dQ's first 64 columns in
  // [64, 128)), dP^T [128, 256) (then dS^T in [128, 192), dQ's columns 64..127
  // in [192, 256) when d = 128), dV [256, 256 + d), dK [256 + d, 256 + 2d)
  const uint32_t col_s = 0, col_dp = 128, col_dv = 256, col_dk = 256 + d;

  auto fail = [&](int where, int info) {
    report_error(err, MSA_ERR_TIMEOUT, kSiteAttnBwd, where, info);
    *abort_flag = 1;
  };
  auto wait_item = [&](int n) -> const BtItem* {
    const int slot = n % kBtItemRing;
    if (!mbar_wait(&ctl->item_full[slot], (n / kBtItemRing) & 1)) {
      fail(n, warp);
      return nullptr;
    }
    return &ctl->ring[slot];
  };

  // P^T, dS^T and dS of the tile's rows [64 half, 64 half + 64) (chunks 2 half
  // and 2 half + 1 of 32 rows): rows 0..63 by warps 4-7, rows 64..127 by
  // warps 8-11 (which also drain).  Each warpgroup stages its own rows'
  // log-sum-exps, sm_scale D and last visible keys first.  A chunk's packed
  // P^T / dS^T go to the first halves of the S^T / dP^T columns, in place:
  // chunks 2 and 3 land on chunk 1's columns, so warps 8-11 store only after
  // warps 4-7 have read chunk 1.
  auto epilogue = [&](int half, int wq, int mt, int tau, int count, int Tb, int Sb, int g, int start,
                      int64_t qrow0, int64_t blk_first) -> bool {
    const int j = 32 * wq + lane;             // this lane's key of the block (TMEM lane)
    const uint32_t lanes = static_cast<uint32_t>(32 * wq) << 16;
    // dS[r][j] in the K-major tile of the dQ product: box j / 64, row r, the
    // 16-byte chunk (j % 64) / 8 swizzled by r % 8, byte 2 (j % 8)
    const uint32_t ds_base = smem_u32(ds_s) + (uint32_t)((j >> 6) * 128 * 128) + (uint32_t)(j & 7) * 2u;
    const uint32_t cin = (uint32_t)((j & 63) >> 3);
    uint32_t swz[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) swz[u] = ((cin ^ (uint32_t)u) & 7u) << 4;
    const int b = tau & 1;
    const int tw = 32 * wq + lane;
    if (tw < 64) {
      const int r0 = 64 * half + tw;
      const int ql = r0 / RQ, hi = r0 - ql * RQ;
      const int idx = mt * qpt + ql;
      int limit = -1;
      float l2 = 0.f, dr = 0.f;
      if (idx < count && hi < Hg) {
        const int64_t t = entries[start + idx] / k;
        const int64_t lim = (int64_t)Sb - Tb + (t - qrow0) - blk_first;
        limit = lim >= kBk - 1 ? kBk - 1 : (int)lim;
        const int64_t row = t * H + (int64_t)g * Hg + hi;
        l2 = lse[row] * 1.4426950408889634f;
        dr = Dg[row] * sm_scale;
      }
      ctl->lse2[b][r0] = l2;
      ctl->dsc[b][r0] = dr;
      ctl->lim[b][r0] = limit;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->rows_ready[half]);
    if (!mbar_wait(&ctl->rows_ready[half], tau & 1) || !mbar_wait(&ctl->s_full, tau & 1)) return false;
    tc_fence_after();
#pragma unroll 1
    for (int cc = 0; cc < 2; ++cc) {
      const int c = 2 * half + cc;
      uint32_t rs[32], rd[32];
      tmem_ld32(tmem + lanes + col_s + 32 * c, rs);
      tmem_ld32(tmem + lanes + col_dp + 32 * c, rd);
      tmem_ld_wait();
      if (half == 0 && cc == 1) {
        // chunk 1's columns are read: warps 8-11 may store over them
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->c1_read);
      }
      const uint32_t lb = smem_u32(&ctl->lse2[b][32 * c]);
      const uint32_t db = smem_u32(&ctl->dsc[b][32 * c]);
      const uint32_t mb = smem_u32(&ctl->lim[b][32 * c]);
      const uint32_t sb = ds_base + (uint32_t)(c * 32 * 128);
      uint32_t pk[16], dk16[16];
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        // four rows' values at a time (every lane reads the same words)
        const float4 l4 = lds_f4(lb + 16 * q4);
        const float4 d4 = lds_f4(db + 16 * q4);
        const int4 m4 = lds_i4(mb + 16 * q4);
        const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
        const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
        const int mv[4] = {m4.x, m4.y, m4.z, m4.w};
        float pp[4], dsv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = 4 * q4 + u;
          // a masked pair gives exact zeros: the tile's unused rows may hold any S and dP
          const bool in = j <= mv[u];
          const float x = fmaf(__uint_as_float(rs[i]), scale_log2, -lv[u]);
          pp[u] = ex2_approx(in ? x : -INFINITY);
          dsv[u] = in ? pp[u] * fmaf(__uint_as_float(rd[i]), sm_scale, -dv[u]) : 0.f;
        }
        pk[2 * q4] = pack_bf16x2(pp[0], pp[1]);
        pk[2 * q4 + 1] = pack_bf16x2(pp[2], pp[3]);
        dk16[2 * q4] = pack_bf16x2(dsv[0], dsv[1]);
        dk16[2 * q4 + 1] = pack_bf16x2(dsv[2], dsv[3]);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = 4 * q4 + u;
          const uint32_t h16 = (dk16[i >> 1] >> (16 * (i & 1))) & 0xffffu;
          st_shared_u16(sb + (uint32_t)(i * 128) + swz[i & 7], h16);
        }
      }
      if (half == 1 && cc == 0) {
        if (!mbar_wait(&ctl->c1_read, tau & 1)) return false;
        tc_fence_after();
      }
      tmem_st16(tmem + lanes + col_s + 16 * c, pk);
      tmem_st16(tmem + lanes + col_dp + 16 * c, dk16);
    }
    tmem_st_wait();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&ctl->p_ready);
    return true;
  };

  if (warp == 0) {
    // ------------------------------------------ scheduler and every load
    int n = 0, tau = 0;
    bool ok = true;
    while (ok) {
      const int slot = n % kBtItemRing;
      if (lane == 0) ok = mbar_wait(&ctl->item_empty[slot], ((n / kBtItemRing) + 1) & 1);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      int it = 0;
      if (lane == 0) it = *abort_flag ? nitems : atomicAdd(ticket, 1);
      it = __shfl_sync(0xffffffffu, it, 0);
      BtItem* R = &ctl->ring[slot];
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
        // the block's keys and values (TMA fills rows past the keys with zeros)
        const int st = n % nkv;
        ok = mbar_wait(&ctl->kv_empty[st], ((n / nkv) + 1) & 1);
        if (ok) {
          uint8_t* kd = kv_s + st * 2 * tile_bytes;
          mbar_arrive_expect_tx(&ctl->kv_full[st], (uint32_t)(2 * tile_bytes));
          for (int h = 0; h < nhalf; ++h) {
            tma_load_3d(kd + h * 128 * 128, &tm_k, &ctl->kv_full[st], 64 * h, I.g, krow);
            tma_load_3d(kd + tile_bytes + h * 128 * 128, &tm_v, &ctl->kv_full[st], 64 * h, I.g, krow);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      const int ntiles = (I.count + qpt - 1) / qpt;
      for (int mt = 0; ok && mt < ntiles; ++mt, ++tau) {
        const int qs = tau % nq;
        if (lane == 0) ok = mbar_wait(&ctl->q_empty[qs], ((tau / nq) + 1) & 1);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        const int nqr = min(qpt, I.count - mt * qpt);
        uint8_t* dst = q_s + qs * 2 * tile_bytes;
        if (lane == 0) mbar_arrive_expect_tx(&ctl->q_full[qs], 2 * nqr * RQ * d * 2);
        __syncwarp();
        const int j = mt * qpt + lane;
        const uint32_t ej = __shfl_sync(0xffffffffu, e0, j & 31);
        const uint32_t ek = __shfl_sync(0xffffffffu, e1, j & 31);
        if (lane < nqr) {
          const int64_t t = (j < 32 ? ej : ek) / k;   // the pass covers every query (t0 = 0)
          const int row = (int)(t * H + (int64_t)I.g * Hg);
          for (int h = 0; h < nhalf; ++h) {
            tma_load_2d(dst + h * 128 * 128 + lane * RQ * 128, &tm_q, &ctl->q_full[qs], 64 * h, row);
            tma_load_2d(dst + tile_bytes + h * 128 * 128 + lane * RQ * 128, &tm_do, &ctl->q_full[qs], 64 * h, row);
          }
        }
        // the next tile's rows into L2 while this one computes (its group's Hg
        // head rows of q and dO, contiguous and inside the tensors)
        if (mt + 1 < ntiles) {
          const int j2 = (mt + 1) * qpt + lane;
          const uint32_t f0 = __shfl_sync(0xffffffffu, e0, j2 & 31);
          const uint32_t f1 = __shfl_sync(0xffffffffu, e1, j2 & 31);
          if (lane < min(qpt, I.count - (mt + 1) * qpt)) {
            const int64_t row2 = (int64_t)((j2 < 32 ? f0 : f1) / k) * H + (int64_t)I.g * Hg;
            prefetch_l2(qg + row2 * d, (uint32_t)(Hg * d * 2));
            prefetch_l2(dog + row2 * d, (uint32_t)(Hg * d * 2));
          }
        }
      }
      if (!ok) break;
      ++n;
    }
    if (lane == 0) {
      if (!ok) fail(n, -1);
      // no load may still be in flight when the CTA exits
      for (int st = 0; st < nkv; ++st) {
        const int issued = n > st ? (n - st + nkv - 1) / nkv : 0;
        if (issued > 0) mbar_wait(&ctl->kv_full[st], (issued - 1) & 1);
      }
      for (int qs = 0; qs < nq; ++qs) {
        const int issued = tau > qs ? (tau - qs + nq - 1) / nq : 0;
        if (issued > 0) mbar_wait(&ctl->q_full[qs], (issued - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t idesc_kv = idesc_bf16_f32(128, d, 0, 1);     // dV, dK: B (dO, Q) MN-major
      const uint32_t idesc_q = idesc_bf16_f32(128, 64, 0, 1);     // dQ, 64 columns: B (K) MN-major
      const uint64_t kmaj_kv = make_sdesc(smem_u32(kv_s), 16, 1024, kSw128);
      const uint64_t kmaj_q = make_sdesc(smem_u32(q_s), 16, 1024, kSw128);
      const uint64_t mn_q = make_sdesc(smem_u32(q_s), 128 * 128, 1024, kSw128);
      const uint64_t mn_kv = make_sdesc(smem_u32(kv_s), 128 * 128, 1024, kSw128);
      const uint64_t kmaj_ds = make_sdesc(smem_u32(ds_s), 16, 1024, kSw128);
      const uint64_t tb16 = (uint64_t)(tile_bytes >> 4);
      int n = 0, tau = 0;
      bool ok = true;
      while (ok && !*abort_flag) {
        const BtItem* R = wait_item(n);
        if (R == nullptr) { ok = false; break; }
        const int cnt = R->count;
        mbar_arrive(&ctl->item_empty[n % kBtItemRing]);
        if (cnt <= 0) break;
        const int st = n % nkv;
        const int ntiles = (cnt + qpt - 1) / qpt;
        const uint64_t kst = (uint64_t)((st * 2 * tile_bytes) >> 4);
        for (int mt = 0; mt < ntiles && ok; ++mt, ++tau) {
          const int qs = tau % nq;
          const uint64_t qst = (uint64_t)((qs * 2 * tile_bytes) >> 4);
          // the tile's rows, the block (first tile), TMEM drained of the previous tile's dQ
          if (!mbar_wait(&ctl->q_full[qs], (tau / nq) & 1) ||
              (mt == 0 && !mbar_wait(&ctl->kv_full[st], (n / nkv) & 1)) ||
              !mbar_wait(&ctl->tmem_free, ((tau & 1) ^ 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          // S^T = K Q^T and dP^T = V dO^T
          for (int kk = 0; kk < d / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4);
            umma_bf16_ss(tmem + col_s, kmaj_kv + kst + off, kmaj_q + qst + off, idesc_s, kk > 0 ? 1u : 0u);
          }
          for (int kk = 0; kk < d / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4);
            umma_bf16_ss(tmem + col_dp, kmaj_kv + kst + tb16 + off, kmaj_q + qst + tb16 + off, idesc_s,
                         kk > 0 ? 1u : 0u);
          }
          umma_commit(&ctl->s_full);
          // P^T and dS^T in TMEM, dS in shared memory; the item's first tile
          // also waits for the previous item's dK and dV to be drained
          if (!mbar_wait(&ctl->p_ready, tau & 1) || (mt == 0 && !mbar_wait(&ctl->dkv_free, ((n & 1) ^ 1)))) {
            ok = false;
            break;
          }
          tc_fence_after();
          // dV += P^T dO and dK += dS^T Q (K = the tile's 128 rows, 16 per step)
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t off = (uint64_t)((kk * 2048) >> 4);
            const uint32_t acc = (mt > 0 || kk > 0) ? 1u : 0u;
            umma_bf16_ts(tmem + col_dv, tmem + col_s + kk * 8, mn_q + qst + tb16 + off, idesc_kv, acc);
            umma_bf16_ts(tmem + col_dk, tmem + col_dp + kk * 8, mn_q + qst + off, idesc_kv, acc);
          }
          // dQ = dS K (K = the block's 128 keys), 64 output columns per product
          for (int h = 0; h < nhalf; ++h) {
            const uint32_t dcol = h == 0 ? col_s + 64 : col_dp + 64;
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t aoff = (uint64_t)(((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4);
              const uint64_t boff = (uint64_t)((h * 128 * 128 + kk * 2048) >> 4);
              umma_bf16_ss(tmem + dcol, kmaj_ds + aoff, mn_kv + kst + boff, idesc_q, kk > 0 ? 1u : 0u);
            }
          }
          umma_commit(&ctl->dq_full);
          umma_commit(&ctl->q_empty[qs]);
          if (mt == ntiles - 1) {
            umma_commit(&ctl->kv_empty[st]);
            umma_commit(&ctl->dkv_full);
          }
        }
        ++n;
      }
      if (!ok) fail(tau, -2);
      umma_commit(&ctl->mma_done);
      mbar_wait(&ctl->mma_done, 0);
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------------------------- P^T, dS^T and dS of rows 0..63
    const int wq = warp & 3;
    int n = 0, tau = 0;
    bool failed = false;
    while (!*abort_flag && !failed) {
      const BtItem* R = wait_item(n);
      if (R == nullptr) break;
      const int count = R->count, Tb = R->Tb, Sb = R->Sb, g = R->g, start = R->start;
      const int64_t qrow0 = R->qrow0;
      const int64_t blk_first = (int64_t)R->blk * kBk;
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->item_empty[n % kBtItemRing]);
      if (count <= 0) break;
      const int ntiles = (count + qpt - 1) / qpt;
      for (int mt = 0; mt < ntiles; ++mt, ++tau) {
        if (!epilogue(0, wq, mt, tau, count, Tb, Sb, g, start, qrow0, blk_first)) {
          fail(tau, 1);
          failed = true;
          break;
        }
      }
      ++n;
    }
  } else if (warp >= 8) {
    // ------------------------------------------------ dQ, dK and dV drains
    const int wq = warp & 3;
    const int r = 32 * wq + lane;             // tile row (dQ) or key (dK, dV) of this lane
    const uint32_t lanes = static_cast<uint32_t>(32 * wq) << 16;
    const int ql = r / RQ, hi = r - ql * RQ;
    int n = 0, tau = 0;
    while (!*abort_flag) {
      const BtItem* R = wait_item(n);
      if (R == nullptr) break;
      const int count = R->count, Tb = R->Tb, Sb = R->Sb, g = R->g, start = R->start;
      const int64_t qrow0 = R->qrow0;
      const int64_t krow = R->krow;
      const int64_t blk_first = (int64_t)R->blk * kBk;
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->item_empty[n % kBtItemRing]);
      if (count <= 0) break;
      const int ntiles = (count + qpt - 1) / qpt;
      bool failed = false;
      for (int mt = 0; mt < ntiles; ++mt, ++tau) {
        if (!epilogue(1, wq, mt, tau, count, Tb, Sb, g, start, qrow0, blk_first)) {
          fail(tau, 4);
          failed = true;
          break;
        }
        const int idx = mt * qpt + ql;
        const bool valid = idx < count && hi < Hg;
        const int64_t row = valid ? (int64_t)(entries[start + idx] / k) * H + (int64_t)g * Hg + hi : 0;
        if (!mbar_wait(&ctl->dq_full, tau & 1)) {
          fail(tau, 2);
          failed = true;
          break;
        }
        tc_fence_after();
        for (int h = 0; h < nhalf; ++h) {
          const uint32_t dcol = h == 0 ? col_s + 64 : col_dp + 64;
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t v[32];
            tmem_ld32(tmem + lanes + dcol + 32 * c, v);
            tmem_ld_wait();
            if (valid) {
              float* dst = dq + row * d + 64 * h + 32 * c;
#pragma unroll
              for (int q4 = 0; q4 < 8; ++q4)
                red_add4(dst + 4 * q4, __uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                         __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ctl->tmem_free);
      }
      if (failed) break;
      // the item's dK and dV: one row per key of the block inside the sequence
      if (!mbar_wait(&ctl->dkv_full, n & 1)) {
        fail(n, 3);
        break;
      }
      tc_fence_after();
      const bool key_ok = blk_first + r < Sb;
      for (int which = 0; which < 2; ++which) {
        float* base = (which == 0 ? dv : dk) + ((krow + r) * G + g) * (int64_t)d;
        const uint32_t col = which == 0 ? col_dv : col_dk;
#pragma unroll 1
        for (int c = 0; c < d / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tmem + lanes + col + 32 * c, v);
          tmem_ld_wait();
          if (key_ok) {
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              red_add4(base + 32 * c + 4 * q4, __uint_as_float(v[4 * q4]), __uint_as_float(v[4 * q4 + 1]),
                       __uint_as_float(v[4 * q4 + 2]), __uint_as_float(v[4 * q4 + 3]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ctl->dkv_free);
      ++n;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kBtTmemCols);
  }
}

// K / V stages and Q / dO slots that fit (d = 64: two of each; d = 128: one).
void bwd_tc_stages(int d, int* nkv, int* nq) {
  const size_t tile = (size_t)128 * d * 2;
  const size_t fixed = 1024 + (size_t)128 * 128 * 2 + sizeof(BtCtl);
  *nkv = 2;
  *nq = 2;
  if (fixed + 8 * tile > kBtSmemLimit) *nkv = 1;
  if (fixed + (size_t)(2 * *nkv + 4) * tile > kBtSmemLimit) *nq = 1;
}

size_t bwd_tc_smem_bytes(int d) {
  int nkv = 0, nq = 0;
  bwd_tc_stages(d, &nkv, &nq);
  return 1024 + (size_t)(nkv + nq) * 2 * 128 * d * 2 + (size_t)128 * 128 * 2 + sizeof(BtCtl);
}

}  // namespace

int launch_sparse_attn_backward_tc(const AttnBwdArgs& a, const AttnArgs& plan, float* Dbuf, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t rows = a.total_q * a.H;
  if (rows <= 0) return 0;
  cudaError_t e = cudaMemsetAsync(a.dq, 0, sizeof(float) * (size_t)rows * a.d, st);
  if (e != cudaSuccess) return (int)e;
  {
    ProfScope p("attn_bwd_rowdot", stream);
    rowdot_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, st>>>(static_cast<const uint16_t*>(a.dout),
                                                                  static_cast<const uint16_t*>(a.out), rows, a.d,
                                                                  Dbuf);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return (int)e;
  int rc = launch_kv_plan(plan, stream);
  if (rc) return rc;
  alignas(64) CUtensorMap tm_k, tm_v, tm_q, tm_do;
  {
    const uint64_t dims[3] = {(uint64_t)a.d, (uint64_t)a.G, (uint64_t)plan.total_k};
    const uint64_t strides[2] = {(uint64_t)a.d * 2, (uint64_t)a.G * a.d * 2};
    const uint32_t box[3] = {64u, 1u, 128u};
    rc = make_tmap_bf16(&tm_k, a.key, 3, dims, strides, box, 128);
    if (rc) return rc;
    rc = make_tmap_bf16(&tm_v, a.value, 3, dims, strides, box, 128);
    if (rc) return rc;
  }
  const int hg = a.H / a.G;
  const int rq = hg <= 8 ? 8 : 16;
  {
    const uint64_t dims[2] = {(uint64_t)a.d, (uint64_t)rows};
    const uint64_t strides[1] = {(uint64_t)a.d * 2};
    const uint32_t box[2] = {64u, (uint32_t)rq};
    rc = make_tmap_bf16(&tm_q, a.q, 2, dims, strides, box, 128);
    if (rc) return rc;
    rc = make_tmap_bf16(&tm_do, a.dout, 2, dims, strides, box, 128);
    if (rc) return rc;
  }
  int nkv = 0, nq = 0;
  bwd_tc_stages(a.d, &nkv, &nq);
  const size_t smem = bwd_tc_smem_bytes(a.d);
  auto kern = rq == 8 ? attn_bwd_items_kernel<8> : attn_bwd_items_kernel<16>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  {
    ProfScope p("attn_bwd", stream);
    kern<<<nsm, kBtThreads, smem, st>>>(tm_k, tm_v, tm_q, tm_do, static_cast<const uint16_t*>(a.q),
                                        static_cast<const uint16_t*>(a.dout), a.lse, Dbuf, plan.items, plan.nitems,
                                        plan.nitems + 1, plan.entries, a.cu_q, a.cu_k, a.H, a.G, a.d, a.k, nkv, nq,
                                        a.sm_scale * 1.4426950408889634f, a.sm_scale, a.dq, a.dk, a.dv, a.err);
  }
  return (int)cudaGetLastError();
}

}  // namespace msa
