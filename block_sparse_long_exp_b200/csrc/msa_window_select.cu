// msa_window_select.cu — the FLOP-matched sliding-window baseline that the MSA
// pages compare the learned selection with: a fixed pattern of the same
// budget, the first n_sink blocks and the most recent ones, with no index
// scores (pnsm.cn "MiniMax Sparse Attention：一篇读懂百万上下文时代的稀疏注意力工程化
// 路线", sec. 6 "Learnable sink 和滑动窗口消融"; yhxrc.cn sec. 三).  Its output has
// the selection layout, so the main-branch calls run it unchanged.
#include <cuda_runtime.h>

#include "msa_common.cuh"
#include "msa_internal.h"
#include "msa_window.h"

namespace msa {
namespace {

constexpr int kWinThreads = 256;

// One thread per (query, group) row.
__global__ void __launch_bounds__(kWinThreads)
window_select_kernel(const int32_t* __restrict__ cu_q, const int32_t* __restrict__ cu_k, int batch, int G, int k,
                     int n_sink, int64_t total_q, int32_t* __restrict__ sel, DevError* err) {
  const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= total_q * G) return;
  const int64_t t = r / G;
  int lo = 0, hi = batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu_q[mid] <= t) lo = mid; else hi = mid;
  }
  const int Tb = cu_q[lo + 1] - cu_q[lo];
  const int Sb = cu_k[lo + 1] - cu_k[lo];
  int32_t* out = sel + r * k;
  if (Tb > Sb) {
    report_error(err, MSA_ERR_DEVICE_CHECK, kSiteWindow, lo, Tb);
    for (int i = 0; i < k; ++i) out[i] = -1;
    return;
  }
  const int64_t pos = (int64_t)Sb - Tb + (t - cu_q[lo]);
  window_blocks(pos / kBk, k, n_sink, out);
}

}  // namespace

int launch_window_select(const int32_t* cu_q, const int32_t* cu_k, int32_t batch, int32_t G, int32_t k,
                         int32_t n_sink, int64_t total_q, int32_t* sel, DevError* err, void* stream) {
  const int64_t rows = total_q * G;
  if (rows <= 0) return 0;
  const int64_t blocks = (rows + kWinThreads - 1) / kWinThreads;
  if (blocks > 0x7fffffffLL) return (int)cudaErrorInvalidValue;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ProfScope p("window_select", stream);
  window_select_kernel<<<(unsigned)blocks, kWinThreads, 0, st>>>(cu_q, cu_k, batch, G, k, n_sink, total_q, sel, err);
  return (int)cudaGetLastError();
}

}  // namespace msa

// ---------------------------------------------------------------------------
// The share of each head's dense causal attention weight that the selected
// tokens hold (the pages report the selection covering most of the Main
// Branch's attention weight; yhxrc.cn sec. 二): with lse_sel the log-sum-exp
// over the selected tokens and lse_all the one over every causal token,
// share = sum_{j in J} softmax_all(s)_j = exp(lse_sel - lse_all).
namespace msa {
namespace {

__global__ void __launch_bounds__(256)
selected_share_kernel(const float* __restrict__ lse_sel, const float* __restrict__ lse_all, int64_t n,
                      float* __restrict__ share) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) share[i] = __expf(lse_sel[i] - lse_all[i]);
}

}  // namespace

int launch_selected_share(const float* lse_sel, const float* lse_all, int64_t n, float* share, void* stream) {
  if (n <= 0) return 0;
  const int64_t blocks = (n + 255) / 256;
  if (blocks > 0x7fffffffLL) return (int)cudaErrorInvalidValue;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ProfScope p("selected_share", stream);
  selected_share_kernel<<<(unsigned)blocks, 256, 0, st>>>(lse_sel, lse_all, n, share);
  return (int)cudaGetLastError();
}

}  // namespace msa
