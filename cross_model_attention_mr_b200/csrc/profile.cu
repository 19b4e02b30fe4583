// Optional per-kernel CUDA-event timing and a process-wide launch counter (measurement only).
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/mr.h"
#include "profile.h"

namespace mr {
namespace {

const char* const kNames[kNumKernelIds] = {
    "mr_compress_stats", "mr_scan_counts", "mr_emit", "mr_retrieve", "mr_dense", "mr_export",
    "mr_compress_tc", "mr_emit_tc", "mr_retrieve_tc", "mr_dense_tc", "mr_wait_probe", "mr_prep", "mr_gather_probe",
};

struct Record {
  int id;
  cudaEvent_t start, stop;
};

std::mutex g_mu;
std::atomic<int> g_on{0};
std::atomic<long long> g_launches{0};
std::vector<Record> g_records;
std::vector<cudaEvent_t> g_pool;
thread_local cudaEvent_t t_pending = nullptr;

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

void prof_begin(int id, cudaStream_t st) {
  (void)id;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (!g_on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_mu);
  t_pending = take_event();
  if (t_pending) cudaEventRecord(t_pending, st);
}

void prof_end(int id, cudaStream_t st) {
  if (!g_on.load(std::memory_order_relaxed) || !t_pending) return;
  std::lock_guard<std::mutex> lk(g_mu);
  cudaEvent_t stop = take_event();
  if (!stop) return;
  cudaEventRecord(stop, st);
  g_records.push_back(Record{id, t_pending, stop});
  t_pending = nullptr;
}

}  // namespace mr

extern "C" {

int mr_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(mr::g_mu);
  const int prev = mr::g_on.exchange(on ? 1 : 0);
  if (on) {
    for (auto& r : mr::g_records) {
      mr::g_pool.push_back(r.start);
      mr::g_pool.push_back(r.stop);
    }
    mr::g_records.clear();
  }
  return prev;
}

int mr_profile_read(double* total_ms, int64_t* launches, int max_ids) {
  std::lock_guard<std::mutex> lk(mr::g_mu);
  const int n = max_ids < mr::kNumKernelIds ? max_ids : mr::kNumKernelIds;
  for (int i = 0; i < n; ++i) {
    if (total_ms) total_ms[i] = 0.0;
    if (launches) launches[i] = 0;
  }
  for (auto& r : mr::g_records) {
    if (r.id < 0 || r.id >= n) continue;
    float ms = 0.f;
    if (cudaEventSynchronize(r.stop) == cudaSuccess && cudaEventElapsedTime(&ms, r.start, r.stop) == cudaSuccess) {
      if (total_ms) total_ms[r.id] += ms;
    }
    if (launches) launches[r.id] += 1;
  }
  return mr::kNumKernelIds;
}

const char* mr_kernel_name(int id) {
  if (id < 0 || id >= mr::kNumKernelIds) return nullptr;
  return mr::kNames[id];
}

int64_t mr_kernel_launches(void) { return mr::g_launches.load(); }

}  // extern "C"
