// msa_policy_select.cu — the Index Branch under a selection policy with forced
// sink blocks and a forced local window (msa_policy_unit.cuh), a first plain
// form on the CUDA cores: one CTA of 128 threads per (query, group); the
// threads score the non-forced causal blocks into shared memory, thread 0
// chooses.  With no sink and a one-block window it is the final rule that
// msa_index_topk computes with tensor cores.
#include <cuda_runtime.h>

#include "msa_common.cuh"
#include "msa_internal.h"
#include "msa_policy.h"
#include "msa_policy_unit.cuh"

namespace msa {
namespace {

constexpr int kPolThreads = 128;

__global__ void __launch_bounds__(kPolThreads)
policy_select_kernel(const uint16_t* __restrict__ q_idx, const uint16_t* __restrict__ k_idx,
                     const int32_t* __restrict__ cu_q, const int32_t* __restrict__ cu_k, int batch, int G,
                     int d_idx, int k, int n_sink, int n_local, int32_t* __restrict__ sel, DevError* err) {
  __shared__ float score[kPolicyMaxBlocks];
  __shared__ float qif[128];
  const int tid = threadIdx.x;
  const int64_t unit = blockIdx.x;
  const int64_t t = unit / G;
  const int g = static_cast<int>(unit - t * G);
  int32_t* out = sel + (t * G + g) * k;
  int lo = 0, hi = batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu_q[mid] <= t) lo = mid; else hi = mid;
  }
  const int Tb = cu_q[lo + 1] - cu_q[lo];
  const int Sb = cu_k[lo + 1] - cu_k[lo];
  const int64_t pos = (int64_t)Sb - Tb + (t - cu_q[lo]);
  const int64_t lb = pos / kBk;
  if (Tb > Sb || lb >= kPolicyMaxBlocks) {
    if (tid == 0) report_error(err, MSA_ERR_DEVICE_CHECK, kSitePolicy, lo, Tb);
    for (int i = tid; i < k; i += kPolThreads) out[i] = -1;
    return;
  }
  for (int i = tid; i < d_idx; i += kPolThreads) qif[i] = pol_bf16(q_idx[(t * G + g) * d_idx + i]);
  __syncthreads();
  const uint16_t* kirow = k_idx + (int64_t)cu_k[lo] * d_idx;
  if (lb + 1 > k)
    for (int64_t b = tid; b <= lb; b += kPolThreads)
      score[b] = pol_forced(b, lb, n_sink, n_local) ? 0.f : pol_block_score(qif, kirow, d_idx, kBk, b, pos);
  __syncthreads();
  if (tid == 0) pol_select(score, lb, k, n_sink, n_local, out);
}

}  // namespace

int launch_policy_select(const void* q_idx, const void* k_idx, const int32_t* cu_q, const int32_t* cu_k,
                         int32_t batch, int32_t G, int32_t d_idx, int32_t k, int32_t n_sink, int32_t n_local,
                         int64_t total_q, int32_t* sel, DevError* err, void* stream) {
  const int64_t units = total_q * G;
  if (units <= 0) return 0;
  if (d_idx > 128 || k > kPolicyMaxK || units > 0x7fffffffLL) return (int)cudaErrorInvalidValue;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ProfScope p("policy_select", stream);
  policy_select_kernel<<<(unsigned)units, kPolThreads, 0, st>>>(
      static_cast<const uint16_t*>(q_idx), static_cast<const uint16_t*>(k_idx), cu_q, cu_k, batch, G, d_idx, k,
      n_sink, n_local, sel, err);
  return (int)cudaGetLastError();
}

}  // namespace msa
