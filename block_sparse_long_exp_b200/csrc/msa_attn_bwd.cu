// msa_attn_bwd.cu — the Main Branch backward: dq, dk, dv of the attention over
// the selected tokens (or every causal token) for an upstream gradient, as
// defined in msa_bwd_unit.cuh.
//
// A plain form on the CUDA cores: one CTA of 128 threads per (query, group)
// stages the group's query heads and upstream gradients, the heads'
// log-sum-exps and D = dO.o (from the forward's output), then walks its
// support in chunks of 64 tokens.  Per chunk: the tokens' key and value rows
// are copied into shared memory with 16-byte loads (rows padded by one word,
// so that threads reading different rows at the same column hit different
// banks); each thread takes two tokens and four heads for P and dS (so every
// shared-memory load feeds several FMAs); each warp adds whole dk / dv rows of
// its tokens (lane l: columns 4l .. 4l + 3 at d = 128) with one vector
// reduction per row; each thread adds the chunk's dS . K to its dq outputs,
// eight columns of one head at a time.  Every row read lies inside the query's
// sequence: a selected block past the query's own is recorded as
// MSA_ERR_DEVICE_CHECK and left out.
#include <cuda_runtime.h>

#include "msa_bwd.h"
#include "msa_bwd_unit.cuh"
#include "msa_common.cuh"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kBwdThreads = 128;
constexpr int kBwdMaxHg = 16;
constexpr int kBwdMaxD = 128;
constexpr int kBwdGroups = kBwdMaxHg * kBwdMaxD / 8 / kBwdThreads;   // 8-column dq groups per thread
constexpr int kBwdRowWords = kBwdMaxD / 2 + 1;               // a staged row: d bf16 and one pad word
static_assert(kBwdThreads == (kBwdChunk / kBwdPdsTokens) * (kBwdMaxHg / kBwdPdsHeads), "token-pair x head-group split");

struct BwdSmem {
  float qf[kBwdMaxHg * kBwdMaxD];
  float dof[kBwdMaxHg * kBwdMaxD];
  float P[kBwdMaxHg * kBwdChunk];
  float dS[kBwdMaxHg * kBwdChunk];
  uint32_t kst[kBwdChunk * kBwdRowWords];
  uint32_t vst[kBwdChunk * kBwdRowWords];
  float ls[kBwdMaxHg];
  float Ds[kBwdMaxHg];
  int64_t first[kBwdMaxBlocks];
  int64_t base[kBwdMaxBlocks + 1];
  int64_t tok[kBwdChunk];
  int nrange;
};

__device__ __forceinline__ void red_add_f32x4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}
__device__ __forceinline__ void red_add_f32x2(float* p, float a, float b) {
  asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(a), "f"(b) : "memory");
}

__global__ void __launch_bounds__(kBwdThreads)
sparse_attn_bwd_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ key,
                       const uint16_t* __restrict__ value, const int32_t* __restrict__ sel,
                       const uint16_t* __restrict__ out, const float* __restrict__ lse,
                       const uint16_t* __restrict__ dout, const int32_t* __restrict__ cu_q,
                       const int32_t* __restrict__ cu_k, int batch, int H, int G, int d, int k, float sm_scale,
                       int dense, float* __restrict__ dq, float* __restrict__ dk, float* __restrict__ dv,
                       DevError* err) {
  extern __shared__ __align__(16) uint8_t bwd_smem_raw[];
  BwdSmem& sm = *reinterpret_cast<BwdSmem*>(bwd_smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t unit = blockIdx.x;
  const int64_t t = unit / G;
  const int g = static_cast<int>(unit - t * G);
  const int Hg = H / G;
  const int rw = d / 2 + 1;                            // words per staged row
  const int64_t row0 = (t * H + (int64_t)g * Hg) * d;   // the group's heads of query t in [T, H, d]
  int lo = 0, hi = batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu_q[mid] <= t) lo = mid; else hi = mid;
  }
  const int Tb = cu_q[lo + 1] - cu_q[lo];
  const int Sb = cu_k[lo + 1] - cu_k[lo];
  if (Tb > Sb) {
    if (tid == 0) report_error(err, MSA_ERR_DEVICE_CHECK, kSiteAttnBwd, lo, Tb);
    for (int i = tid; i < Hg * d; i += kBwdThreads) dq[row0 + i] = 0.f;
    return;
  }
  for (int i = tid; i < Hg * d; i += kBwdThreads) {
    sm.qf[i] = bwd_bf16(q[row0 + i]);
    sm.dof[i] = bwd_bf16(dout[row0 + i]);
  }
  for (int i = tid; i < Hg; i += kBwdThreads) sm.ls[i] = lse[t * H + (int64_t)g * Hg + i];
  __syncthreads();
  for (int h = tid; h < Hg; h += kBwdThreads) {
    float s = 0.f;
    for (int c = 0; c < d; ++c) s += sm.dof[h * d + c] * bwd_bf16(out[row0 + (int64_t)h * d + c]);
    sm.Ds[h] = s;
  }
  const uint16_t* key_seq = key + (int64_t)cu_k[lo] * G * d;
  const uint16_t* val_seq = value + (int64_t)cu_k[lo] * G * d;
  BwdUnit u;
  u.qf = sm.qf;
  u.dof = sm.dof;
  u.lse = sm.ls;
  u.D = sm.Ds;
  u.krow = key_seq;
  u.vrow = val_seq;
  u.blocks = dense ? nullptr : sel + (t * G + g) * k;
  u.nsel = k;
  u.Hg = Hg;
  u.d = d;
  u.G = G;
  u.g = g;
  u.B_k = kBk;
  u.pos = (int64_t)Sb - Tb + (t - cu_q[lo]);
  u.sm_scale = sm_scale;
  u.dense = dense != 0;
  if (tid == 0) {
    int bad = 0;
    sm.nrange = bwd_ranges(u, sm.first, sm.base, &bad);
    if (bad) report_error(err, MSA_ERR_DEVICE_CHECK, kSiteAttnBwd, static_cast<int>(t), g);
  }
  __syncthreads();
  float* dk_seq = dk + (int64_t)cu_k[lo] * G * d;
  float* dv_seq = dv + (int64_t)cu_k[lo] * G * d;
  const int64_t total = sm.base[sm.nrange];
  const int pieces = d / 8;                            // 16-byte pieces per row
  const int cpl = d / 32;                              // dk / dv columns per lane (4 or 2)
  // P / dS tile of this thread: tokens 2 (tid % 32), + 1 and heads 4 (tid / 32) .. + 3
  const int tp = (tid & 31) * kBwdPdsTokens, h0 = (tid >> 5) * kBwdPdsHeads;
  const int nh = Hg - h0 < kBwdPdsHeads ? Hg - h0 : kBwdPdsHeads;
  // dq groups of this thread: group i = tid + i * 128 is head gi / (d / 8), columns 8 (gi % (d / 8)) .. + 7
  const int gpr = d / 8, ngroups = Hg * gpr;
  float acc[kBwdGroups][8];
#pragma unroll
  for (int i = 0; i < kBwdGroups; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[i][e] = 0.f;
  for (int64_t c0 = 0; c0 < total; c0 += kBwdChunk) {
    const int cnt = total - c0 < kBwdChunk ? static_cast<int>(total - c0) : kBwdChunk;
    if (tid < cnt) sm.tok[tid] = bwd_token(sm.first, sm.base, sm.nrange, c0 + tid);
    __syncthreads();
    // the chunk's key and value rows, 16 bytes per load
    for (int i = tid; i < cnt * pieces; i += kBwdThreads) {
      const int s = i / pieces, pc = i - s * pieces;
      const int64_t off = (sm.tok[s] * G + g) * d + pc * 8;
      const uint4 kv = *reinterpret_cast<const uint4*>(key_seq + off);
      const uint4 vv = *reinterpret_cast<const uint4*>(val_seq + off);
      uint32_t* kd = sm.kst + s * rw + pc * 4;
      uint32_t* vd = sm.vst + s * rw + pc * 4;
      kd[0] = kv.x; kd[1] = kv.y; kd[2] = kv.z; kd[3] = kv.w;
      vd[0] = vv.x; vd[1] = vv.y; vd[2] = vv.z; vd[3] = vv.w;
    }
    __syncthreads();
    // P and dS of this thread's tile
    if (tp < cnt && nh > 0)
      bwd_pds(u, sm.kst, sm.vst, rw, tp, cnt - tp < kBwdPdsTokens ? cnt - tp : kBwdPdsTokens, h0, nh, sm.P, sm.dS,
              kBwdChunk);
    __syncthreads();
    // dk / dv: warp w adds the rows of tokens w, w + 4, ...; lane l columns cpl l .. cpl l + cpl - 1
    for (int s = warp; s < cnt; s += kBwdThreads / 32) {
      float gk[4], gv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (e < cpl) bwd_kv_cols(u, sm.P, sm.dS, kBwdChunk, s, lane * cpl + e, &gk[e], &gv[e]);
      const int64_t r = (sm.tok[s] * G + g) * d + lane * cpl;
      if (cpl == 4) {
        red_add_f32x4(dk_seq + r, gk[0], gk[1], gk[2], gk[3]);
        red_add_f32x4(dv_seq + r, gv[0], gv[1], gv[2], gv[3]);
      } else {
        red_add_f32x2(dk_seq + r, gk[0], gk[1]);
        red_add_f32x2(dv_seq + r, gv[0], gv[1]);
      }
    }
#pragma unroll
    for (int i = 0; i < kBwdGroups; ++i) {
      const int gi = tid + i * kBwdThreads;
      if (gi < ngroups) bwd_phase2(u, sm.dS, sm.kst, rw, cnt, gi / gpr, 8 * (gi % gpr), acc[i]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < kBwdGroups; ++i) {
    const int gi = tid + i * kBwdThreads;
    if (gi < ngroups) {
      float* dst = dq + row0 + (int64_t)(gi / gpr) * d + 8 * (gi % gpr);
#pragma unroll
      for (int e = 0; e < 8; ++e) dst[e] = sm_scale * acc[i][e];
    }
  }
}

}  // namespace

int launch_sparse_attn_backward(const AttnBwdArgs& a, void* stream) {
  const int64_t units = a.total_q * a.G;
  if (units <= 0) return 0;
  if (a.H / a.G > kBwdMaxHg || a.d > kBwdMaxD || units > 0x7fffffffLL) return (int)cudaErrorInvalidValue;
  if (a.d % 32 != 0) return (int)cudaErrorInvalidValue;   // whole 16-byte pieces and lanes of 2 or 4 columns
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t smem = sizeof(BwdSmem);
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  ProfScope p("attn_bwd", stream);
  sparse_attn_bwd_kernel<<<(unsigned)units, kBwdThreads, smem, st>>>(
      static_cast<const uint16_t*>(a.q), static_cast<const uint16_t*>(a.key), static_cast<const uint16_t*>(a.value),
      a.sel, static_cast<const uint16_t*>(a.out), a.lse, static_cast<const uint16_t*>(a.dout), a.cu_q, a.cu_k,
      a.batch, a.H, a.G, a.d, a.k, a.sm_scale, a.dense, a.dq, a.dk, a.dv, a.err);
  return (int)cudaGetLastError();
}

}  // namespace msa
