// msa_kl.h — launcher of the index-alignment target kernel (msa_index_kl.cu).
#pragma once

#include <stdint.h>

#include "msa_internal.h"

namespace msa {

constexpr int32_t kSiteIndexKl = 171;   // DevError::where of the index-alignment kernel

struct IndexKlArgs {
  const void* q;       // bf16 [T, H, d]
  const void* key;     // bf16 [S, G, d]
  const void* q_idx;   // bf16 [T, G, d_idx]
  const void* k_idx;   // bf16 [S, d_idx]
  const int32_t* sel;  // [T, G, k]; unused when dense
  const float* lse;    // [T, H] main-branch log-sum-exp over the support
  const int32_t* cu_q;
  const int32_t* cu_k;
  int32_t batch, H, G, d, d_idx, k;
  int64_t total_q;
  float sm_scale, tau;
  int32_t dense;       // 1: the support is every causal token
  float* kl;           // forward out [T, G]
  float* lse_z;        // forward out [T, G] (or null): the student's log-sum-exp; backward in
  float* dq_idx;       // backward out [T, G, d_idx]
  float* dk_idx;       // backward out [S, d_idx] (accumulated: zero it first)
  DevError* err;
};

int launch_index_kl(const IndexKlArgs& a, void* stream);
// Sparse support on the tensor cores (msa_index_kl_tc.cu): `plan` describes
// the KV-outer lists of the whole call (one pass, no query tiles); part holds
// [T, G, k] partials and is zeroed by the call.
int launch_index_kl_tc(const IndexKlArgs& a, const AttnArgs& plan, float4* part, void* stream);
int launch_index_kl_backward(const IndexKlArgs& a, void* stream);
// The gradient on the sparse support over the same plan (msa_index_kl_tc.cu):
// zeroes dq_idx, plans, then adds every item's contributions to dq_idx and
// dk_idx (which the caller has zeroed).
int launch_index_kl_grad_tc(const IndexKlArgs& a, const AttnArgs& plan, void* stream);

}  // namespace msa
