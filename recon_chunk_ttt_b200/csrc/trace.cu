// Optional per-kernel tracing: when enabled, every kernel launch of the
// library is bracketed by two CUDA events recorded on the caller's stream, and
// ttt_trace_read() turns them into launch counts and accumulated device time
// per kernel name.  Disabled (the default), a TraceScope costs one branch.
// Independently, every scope is an NVTX range named after the kernel, so a
// profiler can select the library's launches by range (a no-op without one).

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/ttt.h"
#include "internal.h"

namespace ttt {
namespace {

struct Pending {
  const char* name;
  cudaEvent_t a, b;
};
struct Acc {
  std::string name;
  int64_t launches;
  double ms;
};

std::mutex g_mu;
bool g_on = false;
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_pool;
std::vector<Acc> g_acc;

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

bool trace_on() { return g_on; }

TraceScope::TraceScope(const char* name, cudaStream_t st) : name_(name), st_(st), a_(nullptr) {
  nvtxRangePushA(name);
  if (!g_on) return;
  std::lock_guard<std::mutex> lk(g_mu);
  a_ = take_event();
  if (a_) cudaEventRecord(static_cast<cudaEvent_t>(a_), st_);
}

TraceScope::~TraceScope() {
  nvtxRangePop();
  if (a_ == nullptr) return;
  std::lock_guard<std::mutex> lk(g_mu);
  cudaEvent_t b = take_event();
  if (b == nullptr) {
    g_pool.push_back(static_cast<cudaEvent_t>(a_));
    return;
  }
  cudaEventRecord(b, st_);
  g_pending.push_back({name_, static_cast<cudaEvent_t>(a_), b});
}

}  // namespace ttt

extern "C" {

ttt_status ttt_trace_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(ttt::g_mu);
  ttt::g_on = on != 0;
  return TTT_OK;
}

ttt_status ttt_trace_read(ttt_trace_entry* entries, int32_t capacity, int32_t* count,
                          int32_t reset) {
  if (capacity < 0 || (capacity > 0 && entries == nullptr)) return TTT_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(ttt::g_mu);
  ttt_status st = TTT_OK;
  for (auto& p : ttt::g_pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(p.b) != cudaSuccess || cudaEventElapsedTime(&ms, p.a, p.b) != cudaSuccess)
      st = TTT_ERR_CUDA;
    bool found = false;
    for (auto& a : ttt::g_acc)
      if (a.name == p.name) {
        a.launches += 1;
        a.ms += ms;
        found = true;
        break;
      }
    if (!found) ttt::g_acc.push_back({p.name, 1, (double)ms});
    ttt::g_pool.push_back(p.a);
    ttt::g_pool.push_back(p.b);
  }
  ttt::g_pending.clear();
  const int n = (int)ttt::g_acc.size();
  for (int i = 0; i < n && i < capacity; ++i) {
    std::memset(entries[i].name, 0, sizeof(entries[i].name));
    std::strncpy(entries[i].name, ttt::g_acc[i].name.c_str(), sizeof(entries[i].name) - 1);
    entries[i].launches = ttt::g_acc[i].launches;
    entries[i].total_ms = ttt::g_acc[i].ms;
  }
  if (count) *count = n;
  if (reset) ttt::g_acc.clear();
  return st;
}

}  // extern "C"
