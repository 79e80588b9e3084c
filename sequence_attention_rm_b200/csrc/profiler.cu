// Opt-in per-launch timing: while enabled, every kernel launch of the library
// is bracketed by two CUDA events recorded on the launching stream, so a
// caller can read each kernel's device time without an external profiler.
// Disabled (the default) it costs one atomic load per launch.
#include <atomic>
#include <mutex>
#include <vector>

#include "internal.h"

namespace rm {
namespace prof {

namespace {
struct Rec {
  const char* name;
  cudaEvent_t a, b;
};
std::atomic<bool> g_on{false};
std::mutex g_mu;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

void recycle_all() {
  for (auto& r : g_recs) {
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_recs.clear();
}
}  // namespace

int begin(const char* name, cudaStream_t s) {
  if (!g_on.load(std::memory_order_relaxed)) return -1;
  std::lock_guard<std::mutex> lk(g_mu);
  Rec r{name, take_event(), take_event()};
  if (!r.a || !r.b) return -1;
  cudaEventRecord(r.a, s);
  g_recs.push_back(r);
  return (int)g_recs.size() - 1;
}

void end(int idx, cudaStream_t s) {
  if (idx < 0) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (idx < (int)g_recs.size()) cudaEventRecord(g_recs[idx].b, s);
}

}  // namespace prof
}  // namespace rm

extern "C" {

rm_status rm_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(rm::prof::g_mu);
  rm::prof::recycle_all();
  rm::prof::g_on.store(on != 0);
  return RM_OK;
}

int rm_profile_count(void) {
  std::lock_guard<std::mutex> lk(rm::prof::g_mu);
  return (int)rm::prof::g_recs.size();
}

rm_status rm_profile_get(int i, const char** name, float* ms) {
  std::lock_guard<std::mutex> lk(rm::prof::g_mu);
  if (i < 0 || i >= (int)rm::prof::g_recs.size() || !name || !ms) return RM_ERR_INVALID_ARG;
  const auto& r = rm::prof::g_recs[i];
  if (cudaEventSynchronize(r.b) != cudaSuccess) return RM_ERR_CUDA;
  if (cudaEventElapsedTime(ms, r.a, r.b) != cudaSuccess) return RM_ERR_CUDA;
  *name = r.name;
  return RM_OK;
}

}  // extern "C"
