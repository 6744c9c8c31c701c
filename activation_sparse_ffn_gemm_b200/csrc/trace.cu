// trace.cu — launch counting and optional per-kernel event timing.
//
// Every kernel launch of the library goes through a Launch guard: it bumps a
// process-wide launch counter and, while tracing is enabled, records a CUDA
// event on the launch stream before and after the kernel. twell_trace_collect
// waits for those events and returns each kernel's name and duration, so a
// caller can attribute the time of one call to its kernels without a profiler.
#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "trace.cuh"

namespace twell {

namespace {

struct Rec {
  const char* name;
  cudaEvent_t start, stop;
};

std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_enabled{0};
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

}  // namespace

Launch::Launch(const char* name, cudaStream_t s) : name_(name), s_(s) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (!g_enabled.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_mu);
  start_ = take_event();
  if (start_ && cudaEventRecord(start_, s_) != cudaSuccess) start_ = nullptr;
}

Launch::~Launch() {
  if (!start_) return;
  std::lock_guard<std::mutex> lk(g_mu);
  cudaEvent_t stop = take_event();
  if (stop && cudaEventRecord(stop, s_) == cudaSuccess) g_recs.push_back(Rec{name_, start_, stop});
}

}  // namespace twell

using namespace twell;

extern "C" {

TWELL_API void twell_trace_enable(int on) { g_enabled.store(on ? 1 : 0); }

TWELL_API uint64_t twell_launch_count(void) { return g_launches.load(); }

TWELL_API int twell_trace_collect(twell_trace_rec* out, int max_recs) {
  std::lock_guard<std::mutex> lk(g_mu);
  int n = 0;
  for (const Rec& r : g_recs) {
    float ms = -1.f;
    if (cudaEventSynchronize(r.stop) == cudaSuccess) cudaEventElapsedTime(&ms, r.start, r.stop);
    if (out && n < max_recs) {
      std::memset(out[n].name, 0, sizeof out[n].name);
      std::strncpy(out[n].name, r.name, sizeof out[n].name - 1);
      out[n].ms = ms;
    }
    ++n;
    g_pool.push_back(r.start);
    g_pool.push_back(r.stop);
  }
  g_recs.clear();
  return n;
}

}  // extern "C"
