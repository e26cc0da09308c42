// msa_gather.cu — rows of a paged cache gathered into packed rows, so that a
// prefill (or a chunk of one) over a paged KV cache runs the packed calls
// unchanged: packed row cu_k[b] + j of sequence b is row (page * B_k + j mod
// B_k) of the pages, page = block_table[b, j / B_k].  Rows are opaque byte
// strings (index keys: d_idx bf16; keys or values: G * d bf16), copied 16 bytes
// at a time.  A page outside the cache is recorded as MSA_ERR_DEVICE_CHECK and
// its rows are written as zeros (nothing is read outside the cache).
#include <cuda_runtime.h>

#include "msa_common.cuh"
#include "msa_gather.h"
#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kGatherThreads = 256;

// One CTA per (sequence, block); the threads copy the block's rows as 16-byte
// words.
__global__ void __launch_bounds__(kGatherThreads)
gather_pages_kernel(const int32_t* __restrict__ cu_k, int batch, const int32_t* __restrict__ block_table,
                    int max_blocks, int64_t num_pages, int64_t row_words, const uint4* __restrict__ pages,
                    uint4* __restrict__ packed, int max_blk, DevError* err) {
  const int b = blockIdx.x / max_blk;
  const int j = blockIdx.x - b * max_blk;
  if (b >= batch) return;
  const int Sb = cu_k[b + 1] - cu_k[b];
  const int nrows = Sb - j * kBk < kBk ? Sb - j * kBk : kBk;
  if (nrows <= 0) return;
  int64_t src_row = -1;
  if (j < max_blocks) {
    const int32_t pg = block_table[(int64_t)b * max_blocks + j];
    if (pg >= 0 && pg < num_pages) src_row = gather_src_row(pg, 0, kBk);
  }
  if (src_row < 0 && threadIdx.x == 0) report_error(err, MSA_ERR_DEVICE_CHECK, kSiteGather, b, j);
  const int64_t dst_row = (int64_t)cu_k[b] + (int64_t)j * kBk;
  const int64_t words = (int64_t)nrows * row_words;
  for (int64_t w = threadIdx.x; w < words; w += kGatherThreads)
    packed[dst_row * row_words + w] = src_row >= 0 ? pages[src_row * row_words + w] : make_uint4(0, 0, 0, 0);
}

}  // namespace

int launch_gather_pages(const int32_t* cu_k, int32_t batch, int32_t max_k_len, const int32_t* block_table,
                        int32_t max_blocks, int64_t num_pages, int64_t row_bytes, const void* pages, void* packed,
                        DevError* err, void* stream) {
  if (batch <= 0 || max_k_len <= 0) return 0;
  const int max_blk = (max_k_len + kBk - 1) / kBk;
  const int64_t ctas = (int64_t)batch * max_blk;
  if (ctas > 0x7fffffffLL || row_bytes <= 0 || row_bytes % 16) return (int)cudaErrorInvalidValue;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  ProfScope p("gather_pages", stream);
  gather_pages_kernel<<<(unsigned)ctas, kGatherThreads, 0, st>>>(
      cu_k, batch, block_table, max_blocks, num_pages, row_bytes / 16, static_cast<const uint4*>(pages),
      static_cast<uint4*>(packed), max_blk, err);
  return (int)cudaGetLastError();
}

}  // namespace msa
