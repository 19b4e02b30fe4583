// Exact causal attention on sm_100a (bf16, d = d_v = 128): O = softmax(s) V with
// s_ij = scale * q_i.k_j + b(h, i, j) over keys j <= i ("AttnCache Guide", "The Quadratic
// Self-Attention Cost"), for packed variable-length sequences with a query offset (MapFlow
// section 6, variable-length packing).  It is the reference the method is compared against and
// the path for the rows a receiver does not reuse.
//
// One CTA per (head, 128-row query tile), tiles of the longest sequences first.  Roles:
//   * producer warp: TMA loads of the Q tile and of 128-key K and V tiles into a 2-stage ring
//     (128-byte swizzle);
//   * MMA warp: S_j = Q K_j^T (M = N = 128, K = 128) into one of two Tensor Memory buffers, then,
//     one tile behind, O += P_{j-1} V_{j-1} (P from shared memory, V MN-major) into a third;
//   * one softmax warpgroup, a query row per thread: reads S_j, applies the causal mask and the
//     logit bias, keeps a row reference that moves only when a logit exceeds it by more than 2^8
//     (the accumulator is then rescaled in Tensor Memory), and writes P_j = 2^(s' - reference) as
//     a bf16 128-byte-swizzled operand; at the end it divides O by the row sum and stores it.
// Every wait is bounded (MR_ERR_TIMEOUT, then drain and free Tensor Memory).
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "profile.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace mr {
namespace {

using namespace sm100;

constexpr int kThreads = 256;
constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kSoftmaxWarp0 = 4;  // warps 4..7: warp w reads Tensor Memory lanes 32 (w % 4) ..
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.0f;
constexpr uint32_t kTileBytes = 128 * 128 * 2;

struct Params {
  const int32_t* cu_q;
  const int32_t* cu_k;
  const int32_t* q_offset;
  int n_seq, H, total_q, total_k;
  float a;  // scale * log2(e)
  Bias bias;
  __nv_bfloat16* O;
  WsHeader* ws;
  uint64_t wait_ns;  // limit of the protocol waits (drains keep kTimeoutNs)
  int skip_arrive;   // failure-path test: the softmax withholds its first "P ready" arrive
};

struct Smem {
  __nv_bfloat16 q[2][128 * 64];     // [d half][row][64]
  __nv_bfloat16 k[2][2][128 * 64];  // [stage][d half][key][64]
  __nv_bfloat16 v[2][2][128 * 64];  // [stage][d_v half][key][64]
  __nv_bfloat16 p[2][2][128 * 64];  // [buffer][key half][row][64]
  uint64_t q_full;
  uint64_t k_full[2], v_full[2], kv_empty[2];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[2], p_empty[2];
  uint64_t o_full, mma_done;
  uint32_t tmem_base;
  int abort;
};

struct Tile {
  int seq, t;        // sequence and its 128-row query tile
  int q0, len_q;     // first packed query row of the sequence, its query rows
  int k0;            // first packed key row of the sequence
  int off;           // absolute position of the sequence's first query row
  int nk;            // key tiles the tile needs
};

// The k-th tile in the launch order: the last tile of every sequence, then the second to last,
// and so on (the tiles with the most keys first).  false when k is past the last tile.
__device__ bool find_tile(const Params& p, int k, Tile& tl) {
  for (int r = 0;; ++r) {
    bool any = false;
    for (int s = 0; s < p.n_seq; ++s) {
      const int lq = __ldg(p.cu_q + s + 1) - __ldg(p.cu_q + s);
      const int nt = (lq + 127) / 128;
      if (nt <= r) continue;
      any = true;
      if (k-- == 0) {
        tl.seq = s;
        tl.t = nt - 1 - r;
        tl.q0 = __ldg(p.cu_q + s);
        tl.len_q = lq;
        tl.k0 = __ldg(p.cu_k + s);
        tl.off = p.q_offset ? __ldg(p.q_offset + s) : 0;
        const int last = tl.off + min(tl.t * 128 + 127, lq - 1);  // largest absolute position
        tl.nk = last / 128 + 1;
        return true;
      }
    }
    if (!any) return false;
  }
}

__device__ __forceinline__ void fail(Smem& s, const Params& p, uint32_t detail) {
  set_status(p.ws, MR_ERR_TIMEOUT, detail);
  s.abort = 1;
}

// ------------------------------------------------------------------------------------------------
__device__ void producer(Smem& s, const Params& p, const Tile& tl, int h, const CUtensorMap* tq,
                         const CUtensorMap* tk, const CUtensorMap* tv) {
  if ((threadIdx.x & 31) != 0) return;
  const int qrow = h * p.total_q + tl.q0 + 128 * tl.t;
  mbar_arrive_expect_tx(&s.q_full, kTileBytes);
  tma_load_2d(&s.q[0][0], tq, &s.q_full, 0, qrow);
  tma_load_2d(&s.q[1][0], tq, &s.q_full, 64, qrow);
  int j = 0;
  for (; j < tl.nk; ++j) {
    const int st = j & 1;
    if (j >= 2 && !mbar_wait_sleep(&s.kv_empty[st], ((j >> 1) - 1) & 1, &s.abort, p.wait_ns, 64)) {
      fail(s, p, 0x901);
      break;
    }
    const int krow = h * p.total_k + tl.k0 + 128 * j;
    mbar_arrive_expect_tx(&s.k_full[st], kTileBytes);
    tma_load_2d(&s.k[st][0][0], tk, &s.k_full[st], 0, krow);
    tma_load_2d(&s.k[st][1][0], tk, &s.k_full[st], 64, krow);
    mbar_arrive_expect_tx(&s.v_full[st], kTileBytes);
    tma_load_2d(&s.v[st][0][0], tv, &s.v_full[st], 0, krow);
    tma_load_2d(&s.v[st][1][0], tv, &s.v_full[st], 64, krow);
  }
  // no load may land after the CTA releases its shared memory
  const int never = 0;
  for (int g = j > 2 ? j - 2 : 0; g < j; ++g) {
    mbar_wait(&s.k_full[g & 1], (g >> 1) & 1, &never, kTimeoutNs);
    mbar_wait(&s.v_full[g & 1], (g >> 1) & 1, &never, kTimeoutNs);
  }
  mbar_wait(&s.q_full, 0, &never, kTimeoutNs);
}

// ------------------------------------------------------------------------------------------------
__device__ void mma_issuer(Smem& s, const Params& p, const Tile& tl) {
  if ((threadIdx.x & 31) != 0) return;
  const uint32_t id_qk = idesc_bf16_f32(128, 128, false, false);
  const uint32_t id_pv = idesc_bf16_f32(128, 128, false, true);
  const uint32_t tbase = s.tmem_base;
  const uint32_t o_col = 256;
  bool ok = mbar_wait(&s.q_full, 0, &s.abort, p.wait_ns);
  if (!ok) fail(s, p, 0x911);
  const uint32_t qa[2] = {smem_u32(&s.q[0][0]), smem_u32(&s.q[1][0])};

  // O += P_i V_i once the softmax has written P_i
  auto pv = [&](int i) -> bool {
    const int b = i & 1;
    if (!mbar_wait(&s.p_full[b], (i >> 1) & 1, &s.abort, p.wait_ns) ||
        !mbar_wait(&s.v_full[b], (i >> 1) & 1, &s.abort, p.wait_ns))
      return false;
    tc_fence_after();
    const uint32_t pa[2] = {smem_u32(&s.p[b][0][0]), smem_u32(&s.p[b][1][0])};
    const uint32_t va = smem_u32(&s.v[b][0][0]);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint64_t da = sdesc_sw128(pa[kk >> 2] + 32 * (kk & 3), 16, 1024);
      const uint64_t dv = sdesc_sw128(va + 2048 * kk, 128 * 128, 1024);
      mma_bf16_ss(tbase + o_col, da, dv, id_pv, (i > 0 || kk > 0) ? 1u : 0u);
    }
    mma_commit(&s.p_empty[b]);
    mma_commit(&s.kv_empty[b]);
    return true;
  };

  for (int j = 0; j < tl.nk && ok; ++j) {
    const int b = j & 1;
    if (!mbar_wait(&s.k_full[b], (j >> 1) & 1, &s.abort, p.wait_ns) ||
        (j >= 2 && !mbar_wait(&s.s_empty[b], ((j >> 1) - 1) & 1, &s.abort, p.wait_ns))) {
      fail(s, p, 0x912);
      ok = false;
      break;
    }
    tc_fence_after();
    const uint32_t ka[2] = {smem_u32(&s.k[b][0][0]), smem_u32(&s.k[b][1][0])};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint64_t da = sdesc_sw128(qa[kk >> 2] + 32 * (kk & 3), 16, 1024);
      const uint64_t db = sdesc_sw128(ka[kk >> 2] + 32 * (kk & 3), 16, 1024);
      mma_bf16_ss(tbase + 128 * b, da, db, id_qk, kk > 0 ? 1u : 0u);
    }
    mma_commit(&s.s_full[b]);
    // the previous tile's P V runs while the softmax works on this tile
    if (j >= 1 && !pv(j - 1)) {
      fail(s, p, 0x913);
      ok = false;
    }
  }
  if (ok) {
    if (pv(tl.nk - 1))
      mma_commit(&s.o_full);
    else
      fail(s, p, 0x914);
  }
  // every MMA of this thread completes before Tensor Memory is released
  mma_commit(&s.mma_done);
  const int never = 0;
  mbar_wait(&s.mma_done, 0, &never, kTimeoutNs);
}

// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ float kb_log2(const Bias& b, int h, int j) {
  const float v = kb_term(b, h, j);
  return v == -INFINITY ? 0.f : v * kLog2e;
}

__device__ void softmax_group(Smem& s, const Params& p, const Tile& tl, int h) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q4 = warp & 3;
  const int row = 32 * q4 + lane;                 // row of the query tile
  const int qi = 128 * tl.t + row;                // row within the sequence
  const bool row_ok = qi < tl.len_q;
  const int pos = tl.off + qi;                    // absolute position: keys 0 .. pos
  const uint32_t tbase = s.tmem_base;
  const uint32_t lane_addr = (uint32_t)(32 * q4) << 16;
  const int pos0 = tl.off + 128 * tl.t;           // position of the tile's first row
  float ref = -INFINITY;                          // row reference (base 2)
  float l = 0.f;                                  // row sum of 2^(s' - ref)
  bool ok = true;
  for (int j = 0; j < tl.nk; ++j) {
    const int b = j & 1;
    if (!mbar_wait(&s.s_full[b], (j >> 1) & 1, &s.abort, p.wait_ns)) {
      fail(s, p, 0x921);
      ok = false;
      break;
    }
    tc_fence_after();
    float v[128];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t raw[32];
      tmem_ld32(tbase + lane_addr + 128 * b + 32 * c, raw);
      tmem_wait_ld();
#pragma unroll
      for (int t = 0; t < 32; ++t) v[32 * c + t] = __uint_as_float(raw[t]);
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.s_empty[b]);

    // biased base-2 logits; the causal mask and the sink / window terms only on tiles they touch
    const int j0 = 128 * j;
    const bool special = (j0 + 127 > pos0) || (j0 < p.bias.sink_len) ||
                         (p.bias.window > 0 && j0 + 127 > pos0 - p.bias.window);
    float mt = -INFINITY;
    if (!special) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float o = kb_log2(p.bias, h, j0 + 32 * c);
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          v[32 * c + t] = fmaf(v[32 * c + t], p.a, o);
          mt = fmaxf(mt, v[32 * c + t]);
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float kb = kb_term(p.bias, h, j0 + 32 * c);
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const int key = j0 + 32 * c + t;
          v[32 * c + t] = key <= pos ? fmaf(v[32 * c + t], p.a, bias_with_kb(p.bias, pos, key, kb) * kLog2e)
                                     : -INFINITY;
          mt = fmaxf(mt, v[32 * c + t]);
        }
      }
    }
    if (!row_ok) mt = -INFINITY;
    // move the reference when a logit passes it by more than 2^8; the accumulator of the tiles
    // before is rescaled in Tensor Memory once their P V has completed
    const bool need = mt > ref + kRescale;
    if (__any_sync(0xffffffffu, need)) {
      const float nref = need ? mt : ref;
      const float f = (need && ref != -INFINITY) ? ex2_approx(ref - nref) : (need ? 0.f : 1.f);
      if (j > 0) {
        // P_{j-1} V_{j-1} has completed when its P buffer is released.  That buffer's earlier
        // completion (tile j - 3) was waited for before P_{j-1} was written and tile j + 1's
        // cannot happen before this warpgroup writes P_{j+1}, so the parity names one phase.
        if (!mbar_wait(&s.p_empty[(j - 1) & 1], ((j - 1) >> 1) & 1, &s.abort, p.wait_ns)) {
          fail(s, p, 0x922);
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t xs[32];
          tmem_ld32(tbase + lane_addr + 256 + 32 * c, xs);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) xs[t] = __float_as_uint(__uint_as_float(xs[t]) * f);
          tmem_st32(tbase + lane_addr + 256 + 32 * c, xs);
        }
        tmem_wait_st();
        tc_fence_before();
      }
      l *= f;
      ref = nref;
    }
    // P_j = 2^(s' - ref) as bf16 into the operand buffer this tile uses
    if (j >= 2 && !mbar_wait(&s.p_empty[b], ((j >> 1) - 1) & 1, &s.abort, p.wait_ns)) {
      fail(s, p, 0x923);
      ok = false;
      break;
    }
    const bool live = row_ok && ref != -INFINITY;
    float sum = 0.f;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      char* dst = reinterpret_cast<char*>(&s.p[b][hh][0]) + row * 128;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int x = 64 * hh + 8 * c8 + 2 * e;
          const float p0 = live ? ex2_approx(v[x] - ref) : 0.f;
          const float p1 = live ? ex2_approx(v[x + 1] - ref) : 0.f;
          sum += p0 + p1;
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
          pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        *reinterpret_cast<uint4*>(dst + ((c8 ^ (row & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
    l += sum;
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && !(p.skip_arrive && j == 0)) mbar_arrive(&s.p_full[b]);
  }
  if (!ok) return;
  // epilogue: O / l -> bf16 -> global
  if (!mbar_wait(&s.o_full, 0, &s.abort, p.wait_ns)) {
    fail(s, p, 0x924);
    return;
  }
  tc_fence_after();
  const float inv = (row_ok && l > 0.f) ? 1.f / l : 0.f;
  __nv_bfloat16* orow = p.O + ((size_t)h * p.total_q + tl.q0 + qi) * 128;
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    uint32_t xs[32];
    tmem_ld32(tbase + lane_addr + 256 + 32 * c, xs);
    tmem_wait_ld();
    if (row_ok) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(xs[8 * g + 2 * e]) * inv,
                                                          __uint_as_float(xs[8 * g + 2 * e + 1]) * inv);
          pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        *reinterpret_cast<uint4*>(orow + 32 * c + 8 * g) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
  }
  tc_fence_before();
}

__global__ void __launch_bounds__(kThreads, 1)
    k_dense_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
               const __grid_constant__ CUtensorMap tv, Params p) {
  Tile tl;
  if (!find_tile(p, (int)blockIdx.x, tl)) return;  // past the last tile: the whole CTA leaves
  const int h = (int)blockIdx.y;
  extern __shared__ unsigned char smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&s.q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.k_full[i], 1);
      mbar_init(&s.v_full[i], 1);
      mbar_init(&s.kv_empty[i], 1);
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.s_empty[i], 4);
      mbar_init(&s.p_full[i], 4);
      mbar_init(&s.p_empty[i], 1);
    }
    mbar_init(&s.o_full, 1);
    mbar_init(&s.mma_done, 1);
    s.abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&s.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kProducerWarp)
    producer(s, p, tl, h, &tq, &tk, &tv);
  else if (warp == kMmaWarp)
    mma_issuer(s, p, tl);
  else if (warp >= kSoftmaxWarp0)
    softmax_group(s, p, tl, h);
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(s.tmem_base, 512);
}

}  // namespace

bool tc_dense_supported(const DenseArgs& a) {
  return a.dt == MR_BF16 && a.d == 128 && a.d_v == 128 && a.scale > 0.f &&
         (a.bias.kb == nullptr || a.bias.kb_block % 32 == 0) &&
         (int64_t)a.H * a.total_q < ((int64_t)1 << 31) && (int64_t)a.H * a.total_k < ((int64_t)1 << 31);
}

cudaError_t tc_dense(const DenseArgs& a) {
  Params p;
  p.cu_q = a.cu_q;
  p.cu_k = a.cu_k;
  p.q_offset = a.q_offset;
  p.n_seq = a.n_seq;
  p.H = a.H;
  p.total_q = a.total_q;
  p.total_k = a.total_k;
  p.a = a.scale * kLog2e;
  p.bias = a.bias;
  p.O = (__nv_bfloat16*)a.O;
  p.ws = a.ws;
  debug_waits(&p.wait_ns, &p.skip_arrive);
  if (p.wait_ns == 0) p.wait_ns = kTimeoutNs;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_bf16_2d(&tq, a.Q, 128, (uint64_t)a.H * a.total_q, 256, 64, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tk, a.K, 128, (uint64_t)a.H * a.total_k, 256, 64, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tv, a.V, 128, (uint64_t)a.H * a.total_k, 256, 64, 128)) return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(k_dense_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // an upper bound on the number of 128-row tiles of all sequences; CTAs past the last one leave
  dim3 grid((unsigned)(a.total_q / 128 + a.n_seq), (unsigned)a.H);
  ProfScope ps(kKDenseTc, a.stream);
  k_dense_tc<<<grid, kThreads, smem, a.stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace mr
