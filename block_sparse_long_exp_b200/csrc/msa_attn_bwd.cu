// msa_attn_bwd.cu — the Main Branch backward: dq, dk, dv of the attention over
// the selected tokens (or every causal token) for an upstream gradient, as
// defined in msa_bwd_unit.cuh.
//
// A first, plain form on the CUDA cores: one CTA of 128 threads per (query,
// group) stages the group's query heads and upstream gradients, the heads'
// log-sum-exps and D = dO.o (from the forward's output), then walks its
// support in chunks of 64 tokens: phase 1 (a thread per token) computes dS for
// every head, stages the key row and adds the token's dk / dv rows
// atomically; phase 2 (every thread) adds the chunk's dS . K to its 16 dq
// outputs.  Every row read lies inside the query's sequence: a selected block
// past the query's own is recorded as MSA_ERR_DEVICE_CHECK and left out.
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
constexpr int kBwdOut = kBwdMaxHg * kBwdMaxD / kBwdThreads;   // dq outputs per thread

__global__ void __launch_bounds__(kBwdThreads)
sparse_attn_bwd_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ key,
                       const uint16_t* __restrict__ value, const int32_t* __restrict__ sel,
                       const uint16_t* __restrict__ out, const float* __restrict__ lse,
                       const uint16_t* __restrict__ dout, const int32_t* __restrict__ cu_q,
                       const int32_t* __restrict__ cu_k, int batch, int H, int G, int d, int k, float sm_scale,
                       int dense, float* __restrict__ dq, float* __restrict__ dk, float* __restrict__ dv,
                       DevError* err) {
  __shared__ float qf[kBwdMaxHg * kBwdMaxD];
  __shared__ float dof[kBwdMaxHg * kBwdMaxD];
  __shared__ float ls[kBwdMaxHg];
  __shared__ float Ds[kBwdMaxHg];
  __shared__ float dS[kBwdMaxHg * kBwdChunk];
  __shared__ uint16_t kst[kBwdChunk * kBwdMaxD];
  __shared__ int64_t first[kBwdMaxBlocks];
  __shared__ int64_t base[kBwdMaxBlocks + 1];
  __shared__ int nrange;
  const int tid = threadIdx.x;
  const int64_t unit = blockIdx.x;
  const int64_t t = unit / G;
  const int g = static_cast<int>(unit - t * G);
  const int Hg = H / G;
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
    qf[i] = bwd_bf16(q[row0 + i]);
    dof[i] = bwd_bf16(dout[row0 + i]);
  }
  for (int i = tid; i < Hg; i += kBwdThreads) ls[i] = lse[t * H + (int64_t)g * Hg + i];
  __syncthreads();
  for (int h = tid; h < Hg; h += kBwdThreads) {
    float s = 0.f;
    for (int c = 0; c < d; ++c) s += dof[h * d + c] * bwd_bf16(out[row0 + (int64_t)h * d + c]);
    Ds[h] = s;
  }
  BwdUnit u;
  u.qf = qf;
  u.dof = dof;
  u.lse = ls;
  u.D = Ds;
  u.krow = key + (int64_t)cu_k[lo] * G * d;
  u.vrow = value + (int64_t)cu_k[lo] * G * d;
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
    nrange = bwd_ranges(u, first, base, &bad);
    if (bad) report_error(err, MSA_ERR_DEVICE_CHECK, kSiteAttnBwd, static_cast<int>(t), g);
  }
  __syncthreads();
  float* dk_seq = dk + (int64_t)cu_k[lo] * G * d;
  float* dv_seq = dv + (int64_t)cu_k[lo] * G * d;
  const int64_t total = base[nrange];
  float acc[kBwdOut];
#pragma unroll
  for (int i = 0; i < kBwdOut; ++i) acc[i] = 0.f;
  for (int64_t c0 = 0; c0 < total; c0 += kBwdChunk) {
    const int cnt = total - c0 < kBwdChunk ? static_cast<int>(total - c0) : kBwdChunk;
    if (tid < cnt) {
      const int64_t j = bwd_token(first, base, nrange, c0 + tid);
      bwd_phase1(u, j, tid, dS, kst + tid * d, dk_seq, dv_seq);
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < kBwdOut; ++i) {
      const int o = tid + i * kBwdThreads;
      if (o < Hg * d) acc[i] += bwd_phase2(u, dS, kst, cnt, o);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < kBwdOut; ++i) {
    const int o = tid + i * kBwdThreads;
    if (o < Hg * d) dq[row0 + o] = sm_scale * acc[i];
  }
}

}  // namespace

int launch_sparse_attn_backward(const AttnBwdArgs& a, void* stream) {
  const int64_t units = a.total_q * a.G;
  if (units <= 0) return 0;
  if (a.H / a.G > kBwdMaxHg || a.d > kBwdMaxD || units > 0x7fffffffLL) return (int)cudaErrorInvalidValue;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ProfScope p("attn_bwd", stream);
  sparse_attn_bwd_kernel<<<(unsigned)units, kBwdThreads, 0, st>>>(
      static_cast<const uint16_t*>(a.q), static_cast<const uint16_t*>(a.key), static_cast<const uint16_t*>(a.value),
      a.sel, static_cast<const uint16_t*>(a.out), a.lse, static_cast<const uint16_t*>(a.dout), a.cu_q, a.cu_k,
      a.batch, a.H, a.G, a.d, a.k, a.sm_scale, a.dense, a.dq, a.dk, a.dv, a.err);
  return (int)cudaGetLastError();
}

}  // namespace msa
