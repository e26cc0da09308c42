// Decode of one long sequence split across ranks by key range.  The pages
// select blocks per query by the block scores of the whole cache (pnsm.cn
// explainer sec. 2: top-k with the local block forced; sec. 9: decoding); when
// the cache is cut into key ranges held by different ranks, each rank scores
// only its own blocks.  The global top-(k-1) is within the union of every
// range's own top-(k-1), so:
//   1. each rank takes its range's k-1 best blocks with their scores
//      (msa_index_topk_decode_candidates, msa_decode_index.cu);
//   2. the candidates of all ranks are exchanged and merged under the same
//      order (score descending, lower block id first) with the local block
//      forced (msa_merge_candidates, here): every rank gets the selection the
//      whole cache would give;
//   3. each rank attends only the selected blocks of its own range
//      (msa_select_block_range cuts them out, here; then the decode attention);
//   4. the per-rank normalised outputs are merged by log-sum-exp
//      (msa_combine), as the two-phase combine merges blocks.
#include "msa_common.cuh"

namespace msa {
namespace {

constexpr int kMaxCand = 256;     // candidates per (query, group): ranks x (k - 1)

// Order of the selection: higher score first, then the lower block id (NaN
// ranks as -inf, already so in the candidates).
__device__ __forceinline__ bool ranks_before(float sa, int ia, float sb, int ib) {
  return sa > sb || (sa == sb && ia < ib);
}

__global__ void merge_candidates_kernel(int batch, int G, int k, int n_cand, const int32_t* __restrict__ cand_ids,
                                        const float* __restrict__ cand_scores, const int32_t* __restrict__ local_block,
                                        int32_t* __restrict__ sel, DevError* err) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)batch * G) return;
  const int b = (int)(i / G);
  const int lb = local_block[b];
  const int cap = k - 1;
  float bs[kMaxK];
  int bi[kMaxK];
  int n = 0;
  for (int c = 0; c < n_cand; ++c) {
    const int id = cand_ids[i * n_cand + c];
    if (id < 0) continue;                       // an empty candidate slot
    if (id >= lb) {                             // only blocks before the local one compete
      report_error(err, MSA_ERR_DEVICE_CHECK, kSiteKeySplit, (int)i, id);
      continue;
    }
    float s = cand_scores[i * n_cand + c];
    if (s != s) s = -INFINITY;
    // insert into the sorted list of the best `cap` so far
    int p = n < cap ? n : cap;
    if (p == cap && (cap == 0 || !ranks_before(s, id, bs[cap - 1], bi[cap - 1]))) continue;
    while (p > 0 && ranks_before(s, id, bs[p - 1], bi[p - 1])) {
      if (p < cap) { bs[p] = bs[p - 1]; bi[p] = bi[p - 1]; }
      --p;
    }
    bs[p] = s;
    bi[p] = id;
    if (n < cap) ++n;
  }
  // ascending ids, then the local block, then -1
  for (int a = 1; a < n; ++a) {
    const int v = bi[a];
    int p = a - 1;
    while (p >= 0 && bi[p] > v) { bi[p + 1] = bi[p]; --p; }
    bi[p + 1] = v;
  }
  int32_t* dst = sel + i * k;
  for (int a = 0; a < n; ++a) dst[a] = bi[a];
  dst[n] = lb;
  for (int a = n + 1; a < k; ++a) dst[a] = -1;
}

__global__ void select_range_kernel(int batch, int G, int k, const int32_t* __restrict__ sel,
                                    const int32_t* __restrict__ lo, const int32_t* __restrict__ hi,
                                    int32_t* __restrict__ out) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)batch * G) return;
  const int b = (int)(i / G);
  const int a0 = lo[b], a1 = hi[b];
  int n = 0;
  for (int s = 0; s < k; ++s) {
    const int id = sel[i * k + s];
    if (id >= a0 && id < a1) out[i * k + n++] = id - a0;
  }
  for (; n < k; ++n) out[i * k + n] = -1;
}

}  // namespace
}  // namespace msa

extern "C" msa_status_t msa_merge_candidates(const msa_shape_t* shape, int32_t batch, int32_t n_cand,
                                             const int32_t* cand_ids, const float* cand_scores,
                                             const int32_t* local_block, int32_t* sel, void* ws, size_t ws_bytes,
                                             void* stream) {
  using namespace msa;
  msa_status_t st = check_shape(shape);
  if (st != MSA_OK) return st;
  if (batch < 0 || n_cand < 0 || n_cand > kMaxCand) return MSA_ERR_INVALID_ARG;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ws_bytes < kWsHeader) return MSA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, sizeof(DevError), s) != cudaSuccess) return MSA_ERR_CUDA;
  if (batch == 0) return MSA_OK;
  if (!local_block || !sel || (n_cand > 0 && (!cand_ids || !cand_scores))) return MSA_ERR_INVALID_ARG;
  const int64_t n = (int64_t)batch * shape->G;
  ProfScope ps("merge_candidates", stream);
  merge_candidates_kernel<<<(unsigned)((n + 127) / 128), 128, 0, s>>>(batch, shape->G, shape->k, n_cand, cand_ids,
                                                                    cand_scores, local_block, sel,
                                                                    static_cast<DevError*>(ws));
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}

extern "C" msa_status_t msa_select_block_range(const msa_shape_t* shape, int32_t batch, const int32_t* sel,
                                               const int32_t* blk_lo, const int32_t* blk_hi, int32_t* sel_out,
                                               void* stream) {
  using namespace msa;
  msa_status_t st = check_shape(shape);
  if (st != MSA_OK) return st;
  if (batch < 0) return MSA_ERR_INVALID_ARG;
  if (batch == 0) return MSA_OK;
  if (!sel || !blk_lo || !blk_hi || !sel_out) return MSA_ERR_INVALID_ARG;
  const int64_t n = (int64_t)batch * shape->G;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  ProfScope ps("select_range", stream);
  select_range_kernel<<<(unsigned)((n + 127) / 128), 128, 0, s>>>(batch, shape->G, shape->k, sel, blk_lo, blk_hi,
                                                                sel_out);
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}
