// msa_window.h — the sliding-window baseline's selection rule (host and
// device) and its launcher (msa_window_select.cu).
#pragma once

#include <stdint.h>

#ifndef __CUDACC__
#define MSA_WIN_HD inline
#else
#define MSA_WIN_HD __host__ __device__ __forceinline__
#endif

namespace msa {

struct DevError;
constexpr int32_t kSiteWindow = 181;   // DevError::where of the window selection

// The k blocks of a query whose own block is lb: blocks 0 .. n_sink-1 and the
// k - n_sink most recent ones lb-(k-n_sink)+1 .. lb, ascending; every causal
// block 0 .. lb when there are at most k of them; -1 in the slots left over.
// (0 <= n_sink < k.)
MSA_WIN_HD void window_blocks(int64_t lb, int k, int n_sink, int32_t* out) {
  int n = 0;
  if (lb + 1 <= k) {
    for (int64_t b = 0; b <= lb; ++b) out[n++] = static_cast<int32_t>(b);
  } else {
    for (int b = 0; b < n_sink; ++b) out[n++] = b;
    for (int64_t b = lb - (k - n_sink) + 1; b <= lb; ++b) out[n++] = static_cast<int32_t>(b);
  }
  for (; n < k; ++n) out[n] = -1;
}

int launch_window_select(const int32_t* cu_q, const int32_t* cu_k, int32_t batch, int32_t G, int32_t k,
                         int32_t n_sink, int64_t total_q, int32_t* sel, DevError* err, void* stream);
// share[i] = exp(lse_sel[i] - lse_all[i]) for i < n (msa_window_select.cu).
int launch_selected_share(const float* lse_sel, const float* lse_all, int64_t n, float* share, void* stream);

}  // namespace msa

#undef MSA_WIN_HD
