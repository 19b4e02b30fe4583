// Gather-only measurement kernel for the retrieval's map reads (MapFlow section 5.4: the fused
// kernel streams the kept blocks of every sender head).  It walks a compressed map in the
// retrieval's order -- per 128-row block, key blocks J <= I, the kept tiles of every sender head --
// and moves each kept tile into shared memory with the same mechanism the retrieval's mixers use
// (16-byte cp.async per thread, completion per thread), then discards it.  No arithmetic.  Each
// row block is walked by `readers` CTAs side by side (the retrieval reads a tile once per group of
// receiver heads), so bytes / time gives the gather rate from DRAM (readers = 1) or mostly from L2
// (readers = 16).
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "profile.h"

namespace mr {
namespace {

constexpr int kThreads = 512;
constexpr int kMaxRing = 24;  // 16-byte slots per thread at most (192 KB of shared memory)

__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
    k_gather_probe(const uint32_t* __restrict__ kept_bits, const int32_t* __restrict__ row_ptr, const char* vals,
                   int64_t capacity, int H_s, int nqb, int nkw, int B, int64_t tile_bytes, int readers,
                   int ring_slots, unsigned long long* sink) {
  extern __shared__ uint4 ring_raw[];  // [ring_slots][kThreads] 16-byte slots
  uint4 (*ring)[kThreads] = reinterpret_cast<uint4 (*)[kThreads]>(ring_raw);
  __shared__ uint32_t list[64];
  __shared__ int n_list;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t my = (uint32_t)__cvta_generic_to_shared(&ring[0][tid]);
  const int rows_per_unit = 128 / B;                 // query blocks per 128-row unit
  const int n_rb = (nqb * B + 127) / 128;
  const int n_units = n_rb * readers;
  const int pieces = (int)(tile_bytes / 16);
  uint32_t slot = 0, issued = 0;
  for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
    const int rb = n_rb - 1 - u / readers;           // longest first; the readers of a block together
    for (int qi = 0; qi < rows_per_unit; ++qi) {
      const int I = rb * rows_per_unit + qi;
      if (I >= nqb) continue;
      for (int J = 0; J <= I; ++J) {
        // warp 0 lists the stored tiles (h, I, J) of every sender head
        if (warp == 0) {
          int cnt = 0;
          for (int h0 = 0; h0 < H_s; h0 += 32) {
            const int h = h0 + lane;
            uint32_t t = 0xffffffffu;
            if (h < H_s) {
              const uint32_t* bits = kept_bits + (size_t)(h * nqb + I) * nkw;
              if ((bits[J >> 5] >> (J & 31)) & 1u) {
                const int64_t tt = (int64_t)row_ptr[h * nqb + I] + kept_rank(bits, J);
                if (tt < capacity) t = (uint32_t)tt;
              }
            }
            const uint32_t m = __ballot_sync(0xffffffffu, t != 0xffffffffu);
            if (t != 0xffffffffu) list[cnt + __popc(m & ((1u << lane) - 1u))] = t;
            cnt += __popc(m);
          }
          if (lane == 0) n_list = cnt;
        }
        __syncthreads();
        const int n = n_list;
        for (int k = 0; k < n; ++k) {
          const char* tile = vals + (int64_t)list[k] * tile_bytes;
          for (int pc = tid; pc < pieces; pc += kThreads) {
            cp16(my + slot * (uint32_t)(kThreads * 16), tile + (int64_t)pc * 16);
            slot = slot + 1 == (uint32_t)ring_slots ? 0u : slot + 1;
            // groups of half the ring: at most the whole ring in flight, never a slot reused early
            if (++issued % (uint32_t)(ring_slots / 2) == 0) {
              asm volatile("cp.async.commit_group;" ::: "memory");
              asm volatile("cp.async.wait_group 1;" ::: "memory");
            }
          }
        }
        __syncthreads();
      }
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  // keep the copies observable: one word of the ring per thread into a sink the caller ignores
  atomicAdd(sink, (unsigned long long)ring[0][tid].x);
}

}  // namespace

cudaError_t launch_gather_probe(const mr_bsr& map, int readers, int ring_slots, WsHeader* ws, cudaStream_t st) {
  if (ring_slots < 2 || ring_slots > kMaxRing || ring_slots % 2) return cudaErrorInvalidValue;
  const int nqb = map.L / map.block;
  const int64_t tile_bytes = (int64_t)map.block * map.block * (map.val_dtype == MR_BF16 ? 2 : map.val_dtype == MR_F32 ? 4 : 1);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int n_units = ((map.L + 127) / 128) * readers;
  const int grid = n_units < sms ? n_units : sms;
  const size_t smem = (size_t)ring_slots * kThreads * 16;
  cudaError_t e = cudaFuncSetAttribute(k_gather_probe, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps(kKGatherProbe, st);
  k_gather_probe<<<grid, kThreads, smem, st>>>(map.kept_bits, map.row_ptr, (const char*)map.vals, map.capacity_tiles,
                                            map.H_s, nqb, (nqb + 31) / 32, map.block, tile_bytes, readers,
                                            ring_slots, reinterpret_cast<unsigned long long*>(&ws->counters[0]));
  return cudaGetLastError();
}

}  // namespace mr
