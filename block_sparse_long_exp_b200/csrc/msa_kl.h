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
  float* kl;           // out [T, G]
  DevError* err;
};

int launch_index_kl(const IndexKlArgs& a, void* stream);

}  // namespace msa
