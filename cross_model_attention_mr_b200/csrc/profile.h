// Per-kernel launch accounting (see mr_profile_enable in mr.h).
#pragma once
#include <cuda_runtime.h>

namespace mr {

enum KernelId {
  kKCompressStats = 0,
  kKScanCounts = 1,
  kKEmit = 2,
  kKRetrieve = 3,
  kKDense = 4,
  kKExport = 5,
  kKCompressTc = 6,
  kKEmitTc = 7,
  kKRetrieveTc = 8,
  kKDenseTc = 9,
  kKWaitProbe = 10,
  kKPrep = 11,
  kKGatherProbe = 12,
  kNumKernelIds = 13
};

// Called immediately before and after each kernel launch on `st`.
void prof_begin(int id, cudaStream_t st);
void prof_end(int id, cudaStream_t st);

// RAII bracket around one launch.
struct ProfScope {
  int id;
  cudaStream_t st;
  ProfScope(int i, cudaStream_t s) : id(i), st(s) { prof_begin(id, st); }
  ~ProfScope() { prof_end(id, st); }
};

}  // namespace mr
