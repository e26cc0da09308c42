// msa_bwd.h — launchers of the Main Branch backward kernels (msa_attn_bwd.cu on
// the CUDA cores, msa_attn_bwd_tc.cu on the tensor cores).
#pragma once

#include <stdint.h>

namespace msa {

struct DevError;
struct AttnArgs;
constexpr int32_t kSiteAttnBwd = 191;   // DevError::where of the backward kernel

struct AttnBwdArgs {
  const void* q;       // bf16 [T, H, d]
  const void* key;     // bf16 [S, G, d]
  const void* value;   // bf16 [S, G, d]
  const int32_t* sel;  // [T, G, k]; unused when dense
  const void* out;     // bf16 [T, H, d] the forward's output
  const float* lse;    // [T, H] the forward's log-sum-exp over the support
  const void* dout;    // bf16 [T, H, d] upstream gradient
  const int32_t* cu_q;
  const int32_t* cu_k;
  int32_t batch, H, G, d, k;
  int64_t total_q;
  float sm_scale;
  int32_t dense;       // 1: the support is every causal token
  float* dq;           // out [T, H, d]
  float* dk;           // out [S, G, d] (accumulated: zero it first)
  float* dv;           // out [S, G, d] (accumulated: zero it first)
  DevError* err;
};

int launch_sparse_attn_backward(const AttnBwdArgs& a, void* stream);
// The selected support on the tensor cores (msa_attn_bwd_tc.cu): zeroes dq,
// writes D = dO . O per row into Dbuf [T * H], plans the KV-outer lists of
// `plan` (one pass over every query, no query tiles) and adds every item's
// contributions to dq, dk and dv (dk and dv zeroed by the caller).
int launch_sparse_attn_backward_tc(const AttnBwdArgs& a, const AttnArgs& plan, float* Dbuf, void* stream);

}  // namespace msa
