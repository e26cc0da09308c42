// msa_policy.h — launcher of the selection-policy kernel (msa_policy_select.cu).
#pragma once

#include <stdint.h>

namespace msa {

struct DevError;
constexpr int32_t kSitePolicy = 201;   // DevError::where of the policy selection

int launch_policy_select(const void* q_idx, const void* k_idx, const int32_t* cu_q, const int32_t* cu_k,
                         int32_t batch, int32_t G, int32_t d_idx, int32_t k, int32_t n_sink, int32_t n_local,
                         int64_t total_q, int32_t* sel, DevError* err, void* stream);

}  // namespace msa
