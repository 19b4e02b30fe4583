// mr_compress_noalloc: compression whose scratch comes from a fixed array compiled into libmr.
//
// Some callers cannot allocate device memory at all: code running inside a host framework
// whose pool already owns the GPU's memory (a raw cudaMalloc there fails or fragments that
// pool), plug-ins that must live within a fixed, pre-planned budget, and serving loops that must
// never call the allocator once they are running (an allocation can stall the device).  They
// cannot provide mr_compress's workspace, so this entry point uses the array below instead.  It
// allocates nothing and frees nothing; the caller still provides Q, K and every array of the map.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/mr.h"

namespace {

// The scratch: status header, row normalisers and kept counts of one compression call.  Every
// GPU that loads libmr holds these bytes until the process exits.  All calls share it, and it
// keeps whatever the last call left in it.
static __device__ __align__(256) unsigned char g_compress_scratch[MR_COMPRESS_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// In host code g_compress_scratch names a host-side stand-in, not the device array, so the
// array's device address is looked up once per device, with that device current.
mr_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MR_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MR_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_compress_scratch) != cudaSuccess || addr == nullptr) return MR_ERR_CUDA;
    g_scratch_addr[dev] = addr;
  }
  *out = g_scratch_addr[dev];
  return MR_OK;
}

}  // namespace

extern "C" mr_status mr_compress_noalloc(const void* Q, const void* K, mr_dtype dt, int H_s, int L, int d,
                                         float scale, float p, const mr_logit_bias* bias, mr_bsr* out,
                                         void* stream) {
  if (out == nullptr) return MR_ERR_INVALID_ARG;
  // Reject shapes whose scratch would not fit before touching the device.
  if (mr_compress_workspace_bytes(H_s, L, d, out->block) > (size_t)MR_COMPRESS_NOALLOC_SCRATCH_BYTES)
    return MR_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const mr_status s = scratch_address(&scratch);
  if (s != MR_OK) return s;
  // mr_compress validates everything else, clears the scratch's status header in stream order and
  // overwrites the normalisers and counts before any kernel reads them.
  return mr_compress(Q, K, dt, H_s, L, d, scale, p, bias, out, scratch,
                     (size_t)MR_COMPRESS_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" mr_status mr_compress_noalloc_status(void* stream) {
  void* scratch = nullptr;
  const mr_status s = scratch_address(&scratch);
  if (s != MR_OK) return s;
  // the scratch begins with the status header that the last call's kernels wrote
  return mr_sync_status(scratch, stream);
}
