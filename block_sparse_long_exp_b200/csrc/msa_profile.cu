// Optional per-kernel timing for benchmarks: when enabled, a CUDA event pair is
// recorded on the launch stream around each timed launch; the elapsed times
// are summed per kernel name when read.  Launches are always counted.
#include <cuda_runtime.h>

#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "msa_internal.h"

namespace msa {
namespace {

struct Pending {
  std::string name;
  cudaEvent_t start, stop;
};

std::mutex g_mu;
bool g_enabled = false;
std::vector<Pending> g_pending;
std::map<std::string, std::pair<double, int64_t>> g_done;
std::atomic<int64_t> g_launches{0};

}  // namespace

void prof_count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

ProfScope::ProfScope(const char* name, void* stream) : name_(name), stream_(stream), start_(nullptr), stop_(nullptr) {
  prof_count_launch(1);
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_enabled) return;
  cudaEvent_t a, b;
  if (cudaEventCreate(&a) != cudaSuccess) return;
  if (cudaEventCreate(&b) != cudaSuccess) {
    cudaEventDestroy(a);
    return;
  }
  start_ = a;
  stop_ = b;
  cudaEventRecord(a, reinterpret_cast<cudaStream_t>(stream));
}

ProfScope::~ProfScope() {
  if (start_ == nullptr) return;
  cudaEventRecord(reinterpret_cast<cudaEvent_t>(stop_), reinterpret_cast<cudaStream_t>(stream_));
  std::lock_guard<std::mutex> lk(g_mu);
  g_pending.push_back({name_, reinterpret_cast<cudaEvent_t>(start_), reinterpret_cast<cudaEvent_t>(stop_)});
}

}  // namespace msa

extern "C" {

msa_status_t msa_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(msa::g_mu);
  msa::g_enabled = on != 0;
  return MSA_OK;
}

msa_status_t msa_profile_reset(void) {
  std::lock_guard<std::mutex> lk(msa::g_mu);
  for (auto& p : msa::g_pending) {
    cudaEventSynchronize(p.stop);
    cudaEventDestroy(p.start);
    cudaEventDestroy(p.stop);
  }
  msa::g_pending.clear();
  msa::g_done.clear();
  msa::g_launches.store(0);
  return MSA_OK;
}

msa_status_t msa_profile_read(const char* kernel, double* total_ms, int64_t* count) {
  if (total_ms == nullptr || count == nullptr) return MSA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(msa::g_mu);
  auto& pend = msa::g_pending;
  for (size_t i = 0; i < pend.size(); ++i) {
    float ms = 0.f;
    if (cudaEventSynchronize(pend[i].stop) != cudaSuccess ||
        cudaEventElapsedTime(&ms, pend[i].start, pend[i].stop) != cudaSuccess) {
      pend.erase(pend.begin(), pend.begin() + i);   // keep only the pairs not yet folded in and destroyed
      return MSA_ERR_CUDA;
    }
    auto& slot = msa::g_done[pend[i].name];
    slot.first += ms;
    slot.second += 1;
    cudaEventDestroy(pend[i].start);
    cudaEventDestroy(pend[i].stop);
  }
  pend.clear();
  if (kernel == nullptr) {
    *total_ms = 0.0;
    *count = msa::g_launches.load();
    return MSA_OK;
  }
  auto it = msa::g_done.find(kernel);
  *total_ms = it == msa::g_done.end() ? 0.0 : it->second.first;
  *count = it == msa::g_done.end() ? 0 : it->second.second;
  return MSA_OK;
}

}  // extern "C"
