// msa_gather.h — the paged-cache row map (host and device) and the gather
// launcher (msa_gather.cu).
#pragma once

#include <stdint.h>

#ifndef __CUDACC__
#define MSA_GATHER_HD inline
#else
#define MSA_GATHER_HD __host__ __device__ __forceinline__
#endif

namespace msa {

struct DevError;
constexpr int32_t kSiteGather = 211;   // DevError::where of the page gather

// Row of the pages that holds row r (0 <= r < B_k) of a block stored in page pg.
MSA_GATHER_HD int64_t gather_src_row(int32_t pg, int32_t r, int32_t B_k) {
  return static_cast<int64_t>(pg) * B_k + r;
}

// Packed row of token j of sequence b: cu_k_b + j.  The block it lies in is
// j / B_k, its row in that block j mod B_k.
MSA_GATHER_HD int64_t gather_dst_row(int64_t cu_k_b, int64_t j) { return cu_k_b + j; }

int launch_gather_pages(const int32_t* cu_k, int32_t batch, int32_t max_k_len, const int32_t* block_table,
                        int32_t max_blocks, int64_t num_pages, int64_t row_bytes, const void* pages, void* packed,
                        DevError* err, void* stream);

}  // namespace msa

#undef MSA_GATHER_HD
