// Launch counter and optional per-kernel event timing (for benchmarks and
// profiling; off by default). Timing creates CUDA events on first use of a
// slot and reuses them; it never touches device memory.
#include <atomic>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "launch.cuh"
#include "v4moe_internal.cuh"

namespace v4moe {
namespace {

struct Rec {
  std::string name;
  cudaEvent_t a = nullptr, b = nullptr;
};

std::atomic<bool> g_enabled{false};
std::atomic<unsigned long long> g_launches{0};
std::mutex g_mu;
std::vector<Rec> g_recs;      // recorded (name, start, stop) in launch order
size_t g_used = 0;            // slots in use since the last reset

}  // namespace

bool prof_enabled() { return g_enabled.load(std::memory_order_relaxed); }

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int prof_begin(const char* name, cudaStream_t st) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_used == g_recs.size()) {
    Rec r;
    if (cudaEventCreate(&r.a) != cudaSuccess || cudaEventCreate(&r.b) != cudaSuccess) {
      cudaGetLastError();
      return -1;
    }
    g_recs.push_back(r);
  }
  Rec& r = g_recs[g_used];
  r.name = name;
  cudaEventRecord(r.a, st);
  return int(g_used++);
}

void prof_end(int slot, cudaStream_t st) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (slot >= 0 && size_t(slot) < g_recs.size()) cudaEventRecord(g_recs[size_t(slot)].b, st);
}

}  // namespace v4moe

using namespace v4moe;

extern "C" {

int32_t v4moe_profile_enable(int32_t on) {
  g_enabled.store(on != 0);
  return V4MOE_OK;
}

int32_t v4moe_profile_reset(void) {
  std::lock_guard<std::mutex> lock(g_mu);
  g_used = 0;
  return V4MOE_OK;
}

int32_t v4moe_profile_read(char* names, int32_t name_len, float* total_ms, int32_t* launches,
                           int32_t max_entries, int32_t* n_entries) {
  if (!names || name_len < 2 || !total_ms || !launches || !n_entries || max_entries < 0)
    return V4MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mu);
  std::vector<std::string> keys;
  std::vector<double> ms;
  std::vector<int> cnt;
  for (size_t i = 0; i < g_used; ++i) {
    Rec& r = g_recs[i];
    if (cudaEventSynchronize(r.b) != cudaSuccess) {
      cudaGetLastError();
      return V4MOE_ERR_LAUNCH;
    }
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) {
      cudaGetLastError();
      return V4MOE_ERR_LAUNCH;
    }
    size_t j = 0;
    while (j < keys.size() && keys[j] != r.name) ++j;
    if (j == keys.size()) {
      keys.push_back(r.name);
      ms.push_back(0.0);
      cnt.push_back(0);
    }
    ms[j] += t;
    cnt[j] += 1;
  }
  const int n = int(keys.size() < size_t(max_entries) ? keys.size() : size_t(max_entries));
  for (int i = 0; i < n; ++i) {
    std::strncpy(names + size_t(i) * name_len, keys[size_t(i)].c_str(), size_t(name_len) - 1);
    names[size_t(i) * name_len + name_len - 1] = 0;
    total_ms[i] = float(ms[size_t(i)]);
    launches[i] = cnt[size_t(i)];
  }
  *n_entries = int(keys.size());
  return V4MOE_OK;
}

uint64_t v4moe_launch_count(void) { return g_launches.load(); }

}  // extern "C"
