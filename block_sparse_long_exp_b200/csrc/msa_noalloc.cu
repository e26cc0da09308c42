// Decode-shaped index top-k that allocates nothing: its scratch (the block
// scores, the per-sequence offsets and the device error word) lives in a
// file-scope __device__ array of fixed size instead of a caller workspace.
//
// For callers that cannot allocate device memory when they call in: for
// example a serving loop whose framework reserves all device memory up front
// and hands out no extra buffers, or a host that forbids cudaMalloc on the
// decode path because it synchronizes the device.
#include <cuda_runtime.h>

#include <mutex>

#include "msa_internal.h"

namespace msa {
namespace {

// Every GPU that loads the library holds this array until the process exits.
constexpr size_t kNoAllocScratchBytes = 16u << 20;   // 16 MiB
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the array on the current device, looked up once per
// device (with that device current) and kept for the life of the process.
// Host code must not use the symbol itself as a device pointer: on the host
// it names a stand-in, not device memory.  A cudaDeviceReset unloads the
// module, so the kept address is then stale: the header states that a reset
// ends the use of this entry point on that device.
msa_status_t scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MSA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MSA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MSA_OK;
}

}  // namespace
}  // namespace msa

extern "C" size_t msa_index_topk_decode_noalloc_max_scratch(void) { return msa::kNoAllocScratchBytes; }

extern "C" msa_status_t msa_index_topk_decode_noalloc(const msa_shape_t* shape, const msa_varlen_t* seqs,
                                                      const void* q_idx, const void* k_idx, int32_t* sel,
                                                      int32_t* device_error, void* stream) {
  using namespace msa;
  // the same checks, in the same order, as msa_index_topk
  msa_status_t st = check_shape(shape);
  if (st != MSA_OK) return st;
  st = check_seqs(seqs);
  if (st != MSA_OK) return st;
  if (seqs->max_q_len > 1) return MSA_ERR_INVALID_ARG;          // one query per sequence
  // no queries: nothing is read or written (the data pointers may be NULL)
  if (seqs->total_q > 0 && (q_idx == nullptr || k_idx == nullptr || sel == nullptr)) return MSA_ERR_INVALID_ARG;
  const size_t need = msa_index_topk_workspace_size(shape, seqs);
  if (need == 0) return MSA_ERR_UNSUPPORTED;
  if (need > kNoAllocScratchBytes) return MSA_ERR_WORKSPACE;    // beyond the fixed array
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != MSA_OK) return st;
  // the array keeps the previous call's contents: the error word must start at 0
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, sizeof(DevError), s) != cudaSuccess) return MSA_ERR_CUDA;
  if (seqs->total_q > 0) {
    IndexTopkArgs a{};
    a.q_idx = q_idx; a.k_idx = k_idx; a.sel = sel;
    a.cu_q = seqs->cu_q; a.cu_k = seqs->cu_k;
    a.batch = seqs->batch; a.G = shape->G; a.d_idx = shape->d_idx; a.k = shape->k; a.B_k = shape->B_k;
    a.total_q = seqs->total_q; a.total_k = seqs->total_k;
    a.max_q_len = seqs->max_q_len; a.max_k_len = seqs->max_k_len;
    a.err = static_cast<DevError*>(scratch);
    a.scratch = static_cast<uint8_t*>(scratch) + kWsHeader;
    a.scratch_bytes = kNoAllocScratchBytes - kWsHeader;
    if (launch_index_topk_decode(a, stream) != 0) return MSA_ERR_CUDA;
  }
  if (device_error != nullptr) {
    // copy the device error word's code into the caller's int32 (device memory)
    if (cudaMemcpyAsync(device_error, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return MSA_ERR_CUDA;
  }
  return MSA_OK;
}
