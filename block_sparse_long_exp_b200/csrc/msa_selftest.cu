// Self-test of the bounded waits.  Every spin-wait in the library's kernels
// (an mbarrier phase, a counter that other CTAs advance) gives up after about
// a second and records MSA_ERR_TIMEOUT in the caller's error word, so that a
// wait that can never end (a lost arrival, a failed copy) costs one second and
// an error status instead of a hung GPU.  This kernel makes both kinds of wait
// run out on purpose, on objects that nothing ever signals: an mbarrier that
// nobody arrives on and a counter in the workspace that nobody advances.  The
// waits are the library's own (mbar_wait, flag_wait_geq), given a shorter
// limit; the kernel then returns normally and the context stays usable.
#include "msa_common.cuh"

namespace msa {
namespace {

// Workspace after the error word: the counter nobody advances, then the
// number of waits that ran out.
struct SelfTestWords {
  int32_t never_set;
  int32_t timed_out;
};

__global__ void __launch_bounds__(64) wait_timeout_selftest_kernel(DevError* err, SelfTestWords* words,
                                                                    uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // phase 0 of `bar` completes only when one thread arrives: none does
    if (!mbar_wait(&bar, 0, limit_ns)) {
      report_error(err, MSA_ERR_TIMEOUT, kSiteSelfTest, 0, 0);
      atomicAdd(&words->timed_out, 1);
    }
  } else if (threadIdx.x == 32) {
    // the counter stays 0: no CTA advances it
    if (!flag_wait_geq(&words->never_set, 1, limit_ns)) {
      report_error(err, MSA_ERR_TIMEOUT, kSiteSelfTest, 1, 0);
      atomicAdd(&words->timed_out, 1);
    }
  }
}

}  // namespace
}  // namespace msa

extern "C" size_t msa_selftest_wait_timeout_workspace_size(void) { return msa::kWsHeader + 256; }

extern "C" msa_status_t msa_selftest_wait_timeout(uint32_t limit_us, void* ws, size_t ws_bytes, void* stream) {
  using namespace msa;
  if (limit_us == 0 || limit_us > 1000000u) return MSA_ERR_INVALID_ARG;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 ||
      ws_bytes < msa_selftest_wait_timeout_workspace_size())
    return MSA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // error word and both counters start at zero
  if (cudaMemsetAsync(ws, 0, msa_selftest_wait_timeout_workspace_size(), st) != cudaSuccess) return MSA_ERR_CUDA;
  DevError* err = static_cast<DevError*>(ws);
  SelfTestWords* words = reinterpret_cast<SelfTestWords*>(static_cast<uint8_t*>(ws) + kWsHeader);
  ProfScope ps("selftest_wait", stream);
  wait_timeout_selftest_kernel<<<1, 64, 0, st>>>(err, words, (uint64_t)limit_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? MSA_OK : MSA_ERR_CUDA;
}
