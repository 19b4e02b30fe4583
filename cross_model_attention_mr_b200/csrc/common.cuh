// Shared device-side definitions for the libmr kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mr.h"

namespace mr {

// Workspace header shared by every entry point: a status word and work-queue counters.
struct WsHeader {
  uint32_t status;         // first device-side error (mr_status), 0 = none
  uint32_t detail;         // where it happened (kernel-specific code)
  uint32_t counters[14];   // dynamic work queues (zeroed by the host before each launch)
};
static_assert(sizeof(WsHeader) == 64, "header layout");
constexpr size_t kWsHeaderBytes = 256;
// Retrieval workspace after the header: one progress counter per CTA (pages consumed), read by
// the other CTAs of its schedule group to keep the group together.
constexpr int kMaxProgressCtas = 1024;
constexpr size_t kRetrieveWsBytes = kWsHeaderBytes + kMaxProgressCtas * sizeof(uint32_t);

__device__ __forceinline__ void set_status(WsHeader* ws, uint32_t code, uint32_t detail) {
  if (atomicCAS(&ws->status, 0u, code) == 0u) ws->detail = detail;
}

// Bounds-checked build (libmr_checked.so, compiled with -DMR_CHECKED): the tensor-core kernels
// check the index of every global store, and of every map read whose index comes from device
// data, against the extent the host passed.  A miss records MR_ERR_DEVICE_CHECK with the site's
// code (0xC..) and skips the access.  In the normal build the check is compiled out; the checks
// that are always on (capacity, value offsets and pages) stay in both.
#ifdef MR_CHECKED
constexpr bool kCheckedBuild = true;
__device__ __forceinline__ bool checked(WsHeader* ws, bool ok, uint32_t site) {
  if (!ok) set_status(ws, MR_ERR_DEVICE_CHECK, site);
  return ok;
}
#else
constexpr bool kCheckedBuild = false;
__device__ __forceinline__ bool checked(WsHeader*, bool, uint32_t) { return true; }
#endif

// Logit bias b(h, i, j) for a causal pair j <= i: the largest applicable term, 0 if none.
// (Synthetic stand-in for sink / local-window / retrieval-head structure.)
struct Bias {
  int sink_len;
  float sink_bias;
  int window;
  float window_bias;
  const float* kb;  // [heads][n_kb] or nullptr; -inf = no term
  int kb_block;
  int n_kb;
};

inline Bias make_bias(const mr_logit_bias* b) {
  Bias r{0, 0.f, 0, 0.f, nullptr, 1, 0};
  if (b) {
    r.sink_len = b->sink_len;
    r.sink_bias = b->sink_bias;
    r.window = b->window;
    r.window_bias = b->window_bias;
    r.kb = b->kb_bias;
    r.kb_block = b->kb_block > 0 ? b->kb_block : 1;
    r.n_kb = b->n_kb;
  }
  return r;
}

__device__ __forceinline__ float bias_term(const Bias& b, int h, int i, int j) {
  float best = -INFINITY;
  if (j < b.sink_len) best = b.sink_bias;
  if (i - j < b.window) best = fmaxf(best, b.window_bias);
  if (b.kb != nullptr) best = fmaxf(best, __ldg(b.kb + (size_t)h * b.n_kb + j / b.kb_block));
  return best == -INFINITY ? 0.f : best;
}

// The same rule split for tile kernels: the key-block term kb (already looked up for a chunk of
// keys inside one key block, -inf = none) combined with the sink and window terms of (i, j).
__device__ __forceinline__ float bias_with_kb(const Bias& b, int i, int j, float kb) {
  float best = kb;
  if (j < b.sink_len) best = fmaxf(best, b.sink_bias);
  if (i - j < b.window) best = fmaxf(best, b.window_bias);
  return best == -INFINITY ? 0.f : best;
}

__device__ __forceinline__ float kb_term(const Bias& b, int h, int j) {
  return b.kb == nullptr ? -INFINITY : __ldg(b.kb + (size_t)h * b.n_kb + j / b.kb_block);
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Storage order of a B x B map tile (see mr_bsr.vals): the tile is split into panels of
// 128 bytes of columns (P = 128 / sizeof(T) columns); each panel stores its B rows one after the
// other, 128 bytes per row, and inside a row the 16-byte chunk c sits at chunk position
// c ^ (row % 8).  A panel is therefore exactly a 128-byte-swizzled K-major MMA operand and can be
// read by 8 consecutive rows without shared-memory bank conflicts.
template <typename T>
__host__ __device__ __forceinline__ int tile_offset(int a, int b, int B) {
  constexpr int P = 128 / (int)sizeof(T), E = 16 / (int)sizeof(T);
  const int panel = b / P, c = (b % P) / E;
  return panel * B * P + a * P + ((c ^ (a & 7)) * E) + (b % E);
}

// Inverse of tile_offset: row a and column b of the element stored at offset p.
template <typename T>
__host__ __device__ __forceinline__ void tile_coords(int p, int B, int& a, int& b) {
  constexpr int P = 128 / (int)sizeof(T), E = 16 / (int)sizeof(T);
  const int panel = p / (B * P), rem = p - panel * B * P;
  a = rem / P;
  const int pc = (rem % P) / E;
  b = panel * P + ((pc ^ (a & 7)) * E) + (rem % E);
}

// Storage order of an fp8 (e4m3) tile: panels of 64 columns, rows of 64 bytes, no swizzle; within
// each group of 4 columns the bytes are ordered (0, 2, 1, 3), so one 32-bit word splits into the
// half-precision pairs (0, 1) and (2, 3) with one mask and one shift each.
__host__ __device__ __forceinline__ int fp8_perm4(int c) { return ((c & 1) << 1) | (c >> 1); }
__host__ __device__ __forceinline__ int tile_offset_fp8(int a, int b, int B) {
  return (b >> 6) * B * 64 + a * 64 + ((b & 63) & ~3) + fp8_perm4(b & 3);
}
// Scales per fp8 tile (one per 32-row x 64-column piece) and the index of element (a, b)'s scale.
__host__ __device__ __forceinline__ int fp8_scales_per_tile(int B) { return (B / 32) * (B / 64); }
__host__ __device__ __forceinline__ int fp8_scale_index(int a, int b, int B) {
  return (a >> 5) * (B / 64) + (b >> 6);
}
// Largest finite e4m3 value: a piece's values are stored as value / scale with scale = max / 448.
constexpr float kFp8Max = 448.f;

// Rank of key block J among the kept blocks of one row: number of kept blocks below J.
__device__ __forceinline__ int kept_rank(const uint32_t* bits, int J) {
  int r = 0;
  const int w = J >> 5;
  for (int t = 0; t < w; ++t) r += __popc(bits[t]);
  const uint32_t below = (J & 31) ? (bits[w] & ((1u << (J & 31)) - 1u)) : 0u;
  return r + __popc(below);
}

}  // namespace mr
