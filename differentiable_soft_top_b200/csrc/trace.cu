// trace.cu -- launch counting and optional per-kernel CUDA-event timing.
//
// Every kernel launch in the library goes through a Launch guard.  The guard
// always counts the launch; while tracing is on it also records a CUDA event
// on the launching stream before and after the kernel, so the time each
// kernel spends on the device can be read back without a profiler.
#include <atomic>
#include <cstdio>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "launch.h"

namespace lapsum {

namespace {
std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_trace_on{0};
std::mutex g_mu;
struct Pending {
  const char* name;
  cudaEvent_t a, b;
};
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_pool;
struct Acc {
  uint64_t launches = 0;
  double ms = 0.0;
};
std::map<std::string, Acc> g_acc;

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

void note_launch(int count) { g_launches.fetch_add((uint64_t)count, std::memory_order_relaxed); }

Launch::Launch(const char* name, cudaStream_t st) : name_(name), st_(st) {
  note_launch(1);
  if (!g_trace_on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_mu);
  a_ = take_event();
  b_ = take_event();
  if (a_ && b_) cudaEventRecord(a_, st_);
}

Launch::~Launch() {
  if (!a_ || !b_) return;
  std::lock_guard<std::mutex> lk(g_mu);
  cudaEventRecord(b_, st_);
  g_pending.push_back(Pending{name_, a_, b_});
}

}  // namespace lapsum

using namespace lapsum;

extern "C" {

uint64_t lapsum_launch_count(void) { return g_launches.load(); }

void lapsum_trace_enable(int on) { g_trace_on.store(on ? 1 : 0); }

int lapsum_trace_collect(char* buf, size_t len) {
  std::lock_guard<std::mutex> lk(g_mu);
  for (const Pending& p : g_pending) {
    if (cudaEventSynchronize(p.b) != cudaSuccess) return -1;
    float ms = 0.0f;
    if (cudaEventElapsedTime(&ms, p.a, p.b) != cudaSuccess) return -1;
    Acc& a = g_acc[p.name];
    a.launches += 1;
    a.ms += (double)ms;
    g_pool.push_back(p.a);
    g_pool.push_back(p.b);
  }
  g_pending.clear();
  std::string out = "{";
  bool first = true;
  for (const auto& kv : g_acc) {
    char item[160];
    std::snprintf(item, sizeof(item), "%s\"%s\": [%llu, %.6f]", first ? "" : ", ", kv.first.c_str(),
                  (unsigned long long)kv.second.launches, kv.second.ms);
    out += item;
    first = false;
  }
  out += "}";
  if (!buf || len == 0) return (int)out.size() + 1;  // size query: keep the record
  const size_t w = std::min(len - 1, out.size());
  std::memcpy(buf, out.data(), w);
  buf[w] = '\0';
  g_acc.clear();
  return (int)w;
}

}  // extern "C"
