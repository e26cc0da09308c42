// msa_index_kl.cu — the index-alignment target KL(P || Q) of every (query,
// group): the Main Branch's attention on the support (the teacher) against
// the Index Branch's softmax over the same tokens (the student), as defined
// in msa_kl_unit.cuh (pnsm.cn sec. 4 "KL alignment", sec. 5 "Indexer
// warmup"; yhxrc.cn sec. 二).
//
// A first, plain form on the CUDA cores: one CTA of 128 threads per (query,
// group) stages the group's query heads, its index query and the heads'
// log-sum-exps in shared memory; each thread takes every 128th support token
// and keeps the partial sums of msa_kl_unit.cuh; thread 0 merges them.  Every
// key row read is inside the query's sequence: a selected block id outside
// 0..pos / B_k is recorded as MSA_ERR_DEVICE_CHECK and skipped.
#include <cuda_runtime.h>

#include "msa_common.cuh"
#include "msa_kl.h"
#include "msa_kl_unit.cuh"

namespace msa {
namespace {

constexpr int kKlThreads = 128;
constexpr int kKlMaxHg = 16;
constexpr int kKlMaxD = 128;

__global__ void __launch_bounds__(kKlThreads)
index_kl_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ key, const uint16_t* __restrict__ q_idx,
                const uint16_t* __restrict__ k_idx, const int32_t* __restrict__ sel, const float* __restrict__ lse,
                const int32_t* __restrict__ cu_q, const int32_t* __restrict__ cu_k, int batch, int H, int G, int d,
                int d_idx, int k, float sm_scale, float tau, int dense, float* __restrict__ kl,
                float* __restrict__ lse_z, DevError* err) {
  __shared__ float qf[kKlMaxHg * kKlMaxD];
  __shared__ float qif[kKlMaxD];
  __shared__ float ls[kKlMaxHg];
  __shared__ KlPartial parts[kKlThreads];
  const int64_t unit = blockIdx.x;
  const int64_t t = unit / G;
  const int g = static_cast<int>(unit - t * G);
  const int Hg = H / G;
  int lo = 0, hi = batch;   // sequence b with cu_q[b] <= t < cu_q[b + 1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu_q[mid] <= t) lo = mid; else hi = mid;
  }
  const int Tb = cu_q[lo + 1] - cu_q[lo];
  const int Sb = cu_k[lo + 1] - cu_k[lo];
  if (Tb > Sb) {
    if (threadIdx.x == 0) {
      report_error(err, MSA_ERR_DEVICE_CHECK, kSiteIndexKl, lo, Tb);
      kl[t * G + g] = 0.f;
    }
    return;
  }
  for (int i = threadIdx.x; i < Hg * d; i += blockDim.x) qf[i] = kl_bf16(q[(t * H + (int64_t)g * Hg) * d + i]);
  for (int i = threadIdx.x; i < d_idx; i += blockDim.x) qif[i] = kl_bf16(q_idx[(t * G + g) * d_idx + i]);
  for (int i = threadIdx.x; i < Hg; i += blockDim.x) ls[i] = lse[t * H + (int64_t)g * Hg + i];
  __syncthreads();
  KlUnit u;
  u.qf = qf;
  u.qif = qif;
  u.lse = ls;
  u.krow = key + (int64_t)cu_k[lo] * G * d;
  u.kirow = k_idx + (int64_t)cu_k[lo] * d_idx;
  u.blocks = dense ? nullptr : sel + (t * G + g) * k;
  u.nsel = k;
  u.Hg = Hg;
  u.d = d;
  u.d_idx = d_idx;
  u.G = G;
  u.g = g;
  u.B_k = kBk;
  u.pos = (int64_t)Sb - Tb + (t - cu_q[lo]);
  u.sm_scale = sm_scale;
  u.tau = tau;
  u.dense = dense != 0;
  int bad = 0;
  parts[threadIdx.x] = kl_thread(u, threadIdx.x, blockDim.x, &bad);
  if (bad) report_error(err, MSA_ERR_DEVICE_CHECK, kSiteIndexKl, static_cast<int>(t), g);
  __syncthreads();
  if (threadIdx.x == 0) {
    float lz;
    kl[t * G + g] = kl_merge(parts, blockDim.x, &lz);
    if (lse_z != nullptr) lse_z[t * G + g] = lz;
  }
}

// Gradient with respect to the index query and keys (teacher held constant):
// the same staging, the student's log-sum-exp from the forward, dq summed in
// shared memory, dk added to global memory atomically.
__global__ void __launch_bounds__(kKlThreads)
index_kl_grad_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ key,
                     const uint16_t* __restrict__ q_idx, const uint16_t* __restrict__ k_idx,
                     const int32_t* __restrict__ sel, const float* __restrict__ lse, const float* __restrict__ lse_z,
                     const int32_t* __restrict__ cu_q, const int32_t* __restrict__ cu_k, int batch, int H, int G,
                     int d, int d_idx, int k, float sm_scale, float tau, int dense, float* __restrict__ dq_idx,
                     float* __restrict__ dk_idx, DevError* err) {
  __shared__ float qf[kKlMaxHg * kKlMaxD];
  __shared__ float qif[kKlMaxD];
  __shared__ float ls[kKlMaxHg];
  // each thread's own dq row (stride d_idx + 1: rows start in different banks)
  extern __shared__ float dq_rows[];
  const int rs = d_idx + 1;
  const int64_t unit = blockIdx.x;
  const int64_t t = unit / G;
  const int g = static_cast<int>(unit - t * G);
  const int Hg = H / G;
  int lo = 0, hi = batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu_q[mid] <= t) lo = mid; else hi = mid;
  }
  const int Tb = cu_q[lo + 1] - cu_q[lo];
  const int Sb = cu_k[lo + 1] - cu_k[lo];
  if (Tb > Sb) {
    if (threadIdx.x == 0) report_error(err, MSA_ERR_DEVICE_CHECK, kSiteIndexKl, lo, Tb);
    for (int i = threadIdx.x; i < d_idx; i += blockDim.x) dq_idx[(t * G + g) * d_idx + i] = 0.f;
    return;
  }
  for (int i = threadIdx.x; i < Hg * d; i += blockDim.x) qf[i] = kl_bf16(q[(t * H + (int64_t)g * Hg) * d + i]);
  for (int i = threadIdx.x; i < d_idx; i += blockDim.x) qif[i] = kl_bf16(q_idx[(t * G + g) * d_idx + i]);
  for (int i = threadIdx.x; i < Hg; i += blockDim.x) ls[i] = lse[t * H + (int64_t)g * Hg + i];
  for (int i = 0; i < d_idx; ++i) dq_rows[threadIdx.x * rs + i] = 0.f;
  __syncthreads();
  KlUnit u;
  u.qf = qf;
  u.qif = qif;
  u.lse = ls;
  u.krow = key + (int64_t)cu_k[lo] * G * d;
  u.kirow = k_idx + (int64_t)cu_k[lo] * d_idx;
  u.blocks = dense ? nullptr : sel + (t * G + g) * k;
  u.nsel = k;
  u.Hg = Hg;
  u.d = d;
  u.d_idx = d_idx;
  u.G = G;
  u.g = g;
  u.B_k = kBk;
  u.pos = (int64_t)Sb - Tb + (t - cu_q[lo]);
  u.sm_scale = sm_scale;
  u.tau = tau;
  u.dense = dense != 0;
  int bad = 0;
  kl_grad_thread(u, lse_z[t * G + g], threadIdx.x, blockDim.x, dq_rows + threadIdx.x * rs,
                 dk_idx + (int64_t)cu_k[lo] * d_idx, &bad);
  if (bad) report_error(err, MSA_ERR_DEVICE_CHECK, kSiteIndexKl, static_cast<int>(t), g);
  __syncthreads();
  // dq: the threads' rows summed in thread order
  for (int i = threadIdx.x; i < d_idx; i += blockDim.x) {
    float acc = 0.f;
    for (int r = 0; r < kKlThreads; ++r) acc += dq_rows[r * rs + i];
    dq_idx[(t * G + g) * d_idx + i] = acc;
  }
}

}  // namespace

int launch_index_kl(const IndexKlArgs& a, void* stream) {
  const int64_t units = a.total_q * a.G;
  if (units <= 0) return 0;
  if (a.H / a.G > kKlMaxHg || a.d > kKlMaxD || a.d_idx > kKlMaxD || units > 0x7fffffffLL)
    return (int)cudaErrorInvalidValue;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ProfScope p("index_kl", stream);
  index_kl_kernel<<<(unsigned)units, kKlThreads, 0, st>>>(
      static_cast<const uint16_t*>(a.q), static_cast<const uint16_t*>(a.key), static_cast<const uint16_t*>(a.q_idx),
      static_cast<const uint16_t*>(a.k_idx), a.sel, a.lse, a.cu_q, a.cu_k, a.batch, a.H, a.G, a.d, a.d_idx, a.k,
      a.sm_scale, a.tau, a.dense, a.kl, a.lse_z, a.err);
  return (int)cudaGetLastError();
}

int launch_index_kl_backward(const IndexKlArgs& a, void* stream) {
  const int64_t units = a.total_q * a.G;
  if (units <= 0) return 0;
  if (a.H / a.G > kKlMaxHg || a.d > kKlMaxD || a.d_idx > kKlMaxD || units > 0x7fffffffLL)
    return (int)cudaErrorInvalidValue;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t smem = sizeof(float) * kKlThreads * (a.d_idx + 1);
  const cudaError_t e =
      cudaFuncSetAttribute(index_kl_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  ProfScope p("index_kl_grad", stream);
  index_kl_grad_kernel<<<(unsigned)units, kKlThreads, smem, st>>>(
      static_cast<const uint16_t*>(a.q), static_cast<const uint16_t*>(a.key), static_cast<const uint16_t*>(a.q_idx),
      static_cast<const uint16_t*>(a.k_idx), a.sel, a.lse, a.lse_z, a.cu_q, a.cu_k, a.batch, a.H, a.G, a.d, a.d_idx,
      a.k, a.sm_scale, a.tau, a.dense, a.dq_idx, a.dk_idx, a.err);
  return (int)cudaGetLastError();
}

}  // namespace msa
