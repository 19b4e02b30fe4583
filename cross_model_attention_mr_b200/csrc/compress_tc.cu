// Block top-p compression statistics on sm_100a (bf16 Q/K, d = 128): MapFlow sections 4 and 5.2.
//
// For every (sender head h, 128-row query unit) the kernel computes, in ONE pass over the causal
// key tiles, the row log-normalisers, the block masses
//     M_IJ = (1/n_I) sum_{i in I} sum_{j in J} exp(s_ij) / sum_j exp(s_ij),
// and the top-p selection of each query block, without ever forming the L x L map.
//
// Pipeline (one CTA per SM, persistent, units longest-first):
//   * producer warp: TMA loads of the unit's Q rows and a ring of 128-key K tiles (128-byte
//     swizzle, K-major);
//   * MMA warp: S = Q K^T for one 128 x 128 tile per tcgen05.mma group into one of two Tensor
//     Memory buffers;
//   * two softmax warpgroups take alternate tiles; each thread owns one query row.  For every key
//     block it keeps x_iJ = sum_{j in J} 2^(s'_ij - c_i) in its own Tensor Memory column, where
//     s' is the logit in base 2 and c_i a per-row reference that only moves when a new value
//     exceeds it by more than 2^8 (the stored sums are then rescaled).  So the map is summarised
//     by one number per (row, key block) and Q K^T is computed once;
//   * epilogue: the two warpgroups merge their references and sums into the row normaliser,
//     normalise the stored block sums, reduce them over the rows of each query block (block
//     masses), and select the kept blocks (rank by mass, ties to the smaller block, fp64 prefix
//     sum until p is reached).
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

constexpr int kThreads = 384;
constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kSoftmaxWarp0 = 4;  // warpgroup w = warps 4 + 4w .. 7 + 4w
// Warpgroup 0 (producer, MMA warp, two idle warps) drops to 56 registers so the two softmax
// warpgroups can rise to 224: each SM sub-partition holds one warp of each warpgroup, and
// 56 + 2 x 224 is exactly the launch's 3 x 168.
constexpr int kLaunchRegs = 168;
constexpr int kRegsControl = 56;
constexpr int kRegsSoftmax = 224;
static_assert(kRegsControl + 2 * kRegsSoftmax == 3 * kLaunchRegs, "register split");
constexpr int kKStages = 4;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescale = 8.0f;  // move the row reference only for a jump of more than 2^8
constexpr float kRescaleSum = 256.0f;  // 2^kRescale

struct Params {
  int H, L, B, nqb, nkw, n_rb, n_units;
  int rb_hi;     // units cover 128-row blocks rb_hi - n_rb .. rb_hi - 1
  int qb0, qb1;  // query blocks whose selection is written
  int renorm;    // stored rows are divided by their kept mass (the emit's normaliser absorbs it)
  float a;  // logit scale in base 2: scale * log2(e)
  float p;
  Bias bias;
  float* lse_ws;
  int* count_ws;
  uint32_t* kept_bits;
  float* kept_mass;
  float* mass_out;
  float* lse_out;
  WsHeader* ws;
};

struct Smem {
  __nv_bfloat16 q[2][128 * 64];
  __nv_bfloat16 k[kKStages][2][128 * 64];
  float red[2][4][128];      // per warpgroup, per warp: column partial sums
  float mass[2][256];        // per query block of the unit
  float cref[2][128];        // per warpgroup, per row: reference
  float csum[2][128];        // per warpgroup, per row: partial row sum
  int sorted[2][256];
  uint32_t bits[2][8];
  int kstar[2];
  float kmass[2];
  uint64_t q_full, q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t s_full[2], s_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  int sm_fail;  // written by softmax warps only in tile loops, read between two epilogue barriers
};

__device__ __forceinline__ void fail(Smem& s, const Params& p, uint32_t detail) {
  set_status(p.ws, MR_ERR_TIMEOUT, detail);
  s.abort = 1;
}

// Unit k of the launch: heads in groups of kHeadGroup, each group's row blocks longest first,
// the group's heads side by side.  The CTAs running at one time then share the K rows of a few
// heads, which stay in L2, instead of streaming every head's K from DRAM for each row block.
constexpr int kHeadGroup = 4;
__device__ __forceinline__ void unit_of(const Params& p, int k, int& h, int& rb) {
  const int per_group = kHeadGroup * p.n_rb;
  const int g = k / per_group, rem = k - g * per_group;
  const int hg = min(kHeadGroup, p.H - g * kHeadGroup);  // heads in this group (the last may be short)
  rb = p.rb_hi - 1 - rem / hg;
  h = g * kHeadGroup + rem % hg;
}

// ------------------------------------------------------------------------------------------------
__device__ void producer(Smem& s, const Params& p, const CUtensorMap* tq, const CUtensorMap* tk) {
  const int lane = threadIdx.x & 31;
  if (lane != 0) return;
  uint32_t nk = 0, nu = 0;
  bool ok = true;
  for (int k = blockIdx.x; k < p.n_units && ok; k += gridDim.x, ++nu) {
    int h, rb;
    unit_of(p, k, h, rb);
    if (nu > 0 && !mbar_wait(&s.q_empty, (nu - 1) & 1, &s.abort, kTimeoutNs)) {
      fail(s, p, 0x401);
      ok = false;
      break;
    }
    const int qrow = h * p.L + 128 * rb;
    mbar_arrive_expect_tx(&s.q_full, 2 * 128 * 64 * 2);
    tma_load_2d(&s.q[0][0], tq, &s.q_full, 0, qrow);
    tma_load_2d(&s.q[1][0], tq, &s.q_full, 64, qrow);
    for (int T = 0; T <= rb; ++T, ++nk) {
      const int st = (int)(nk % kKStages);
      if (nk >= (uint32_t)kKStages && !mbar_wait(&s.k_empty[st], ((nk / kKStages) - 1) & 1, &s.abort, kTimeoutNs)) {
        fail(s, p, 0x402);
        ok = false;
        break;
      }
      const int krow = h * p.L + 128 * T;
      mbar_arrive_expect_tx(&s.k_full[st], 2 * 128 * 64 * 2);
      tma_load_2d(&s.k[st][0][0], tk, &s.k_full[st], 0, krow);
      tma_load_2d(&s.k[st][1][0], tk, &s.k_full[st], 64, krow);
    }
  }
  // drain in-flight loads before shared memory can be released
  const int never = 0;
  for (uint32_t g = (nk > (uint32_t)kKStages ? nk - kKStages : 0); g < nk; ++g)
    mbar_wait(&s.k_full[g % kKStages], (g / kKStages) & 1, &never, kTimeoutNs);
  if (nu > 0) mbar_wait(&s.q_full, (nu - 1) & 1, &never, kTimeoutNs);
}

// ------------------------------------------------------------------------------------------------
__device__ void mma_issuer(Smem& s, const Params& p) {
  const int lane = threadIdx.x & 31;
  if (lane != 0) return;
  const uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
  const uint32_t tbase = s.tmem_base;
  uint32_t nk = 0, nu = 0, nb[2] = {0, 0};
  bool ok = true;
  for (int k = blockIdx.x; k < p.n_units && ok; k += gridDim.x, ++nu) {
    int h, rb;
    unit_of(p, k, h, rb);
    if (!mbar_wait(&s.q_full, nu & 1, &s.abort, kTimeoutNs)) {
      fail(s, p, 0x411);
      break;
    }
    for (int T = 0; T <= rb; ++T, ++nk) {
      const int st = (int)(nk % kKStages), b = T & 1;
      if (!mbar_wait(&s.k_full[st], (nk / kKStages) & 1, &s.abort, kTimeoutNs) ||
          (nb[b] > 0 && !mbar_wait(&s.s_empty[b], (nb[b] - 1) & 1, &s.abort, kTimeoutNs))) {
        fail(s, p, 0x412);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t qa[2] = {smem_u32(&s.q[0][0]), smem_u32(&s.q[1][0])};
      const uint32_t ka[2] = {smem_u32(&s.k[st][0][0]), smem_u32(&s.k[st][1][0])};
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t da = sdesc_sw128(qa[kk >> 2] + 32 * (kk & 3), 16, 1024);
        const uint64_t db = sdesc_sw128(ka[kk >> 2] + 32 * (kk & 3), 16, 1024);
        mma_bf16_ss(tbase + 128 * b, da, db, idesc, kk > 0 ? 1u : 0u);
      }
      mma_commit(&s.s_full[b]);
      mma_commit(&s.k_empty[st]);
      ++nb[b];
    }
    if (ok) mma_commit(&s.q_empty);
  }
  mma_commit(&s.mma_done);
  const int never = 0;
  mbar_wait(&s.mma_done, 0, &never, kTimeoutNs);
}

// ------------------------------------------------------------------------------------------------
// Softmax warpgroups
// ------------------------------------------------------------------------------------------------
// Maximum of 32 values as a tree (short dependency chains).
__device__ __forceinline__ float warp_max32(const float (&v)[32]) {
  float m[16];
#pragma unroll
  for (int t = 0; t < 16; ++t) m[t] = fmaxf(v[t], v[t + 16]);
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
    for (int t = 0; t < w; ++t) m[t] = fmaxf(m[t], m[t + w]);
  return m[0];
}

// Sum of 2^x over 32 values with 8 independent partial sums.  The values kEmuMask names (bit k:
// value 8 m + k) take the FMA-pipe exponential of degree 5, the rest the multi-function unit.
// None do: with the exponentials taken before the max (most tiles need no max pass), the kernel is
// no longer bound by the multi-function unit, and moving 1 or 2 of every 8 measured slower.
constexpr uint32_t kEmuMask = 0x00;
__device__ __forceinline__ float ex2_mixed(float x, int t) {
  return ((kEmuMask >> (t & 7)) & 1) ? ex2_poly<5>(x) : ex2_approx(x);
}
__device__ __forceinline__ float sum_ex2_32(const float (&x)[32]) {
  float a[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) a[t] = ex2_mixed(x[t], t);
#pragma unroll
  for (int t = 8; t < 32; ++t) a[t & 7] += ex2_mixed(x[t], t);
  return ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
}

// Base-2 bias offset of key j for head h when only the key-block term can apply.
__device__ __forceinline__ float kb_offset(const Bias& b, int h, int j) {
  if (b.kb == nullptr) return 0.f;
  const float v = __ldg(b.kb + (size_t)h * b.n_kb + j / b.kb_block);
  return v == -INFINITY ? 0.f : v * kLog2e;
}

__device__ void softmax_group(Smem& s, const Params& p, int w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q4 = warp & 3;                 // lane quarter of Tensor Memory this warp may access
  const int row = 32 * q4 + lane;          // query row within the unit
  const int gtid = threadIdx.x - 32 * (kSoftmaxWarp0 + 4 * w);  // 0..127 within the warpgroup
  const uint32_t tbase = s.tmem_base;
  const uint32_t lane_addr = (uint32_t)(32 * q4) << 16;
  const uint32_t xbase = 256 + 128 * w;    // this warpgroup's block-sum columns
  const int per_tile = p.B == 128 ? 1 : 2; // block-sum columns per 128-key tile
  uint32_t nb = 0;
  bool ok = true;
  for (int k = blockIdx.x; k < p.n_units && ok; k += gridDim.x) {
    int h, rb;
    unit_of(p, k, h, rb);
    const int i = 128 * rb + row;          // absolute query position of this thread's row
    const bool row_ok = i < p.L;
    float c = -INFINITY;                   // row reference (base 2)
    int used = 0;                          // block-sum columns written in this unit
    for (int T = w; T <= rb; T += 2) {
      // the key-block bias terms of this tile (one per 32 keys), fetched before the wait for S so
      // their latency hides behind the MMA
      float kbo[4];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) kbo[cc] = kb_offset(p.bias, h, 128 * T + 32 * cc);
      if (!mbar_wait(&s.s_full[w], nb & 1, &s.abort, kTimeoutNs)) {
        // Leave the tile loop but still pass the epilogue's barriers of this unit: the other
        // warpgroup's bounded waits see the abort flag and meet us there.
        fail(s, p, 0x421);
        s.sm_fail = 1;
        ok = false;
        break;
      }
      ++nb;
      tc_fence_after();
      const int j_tile = 128 * T;
      const bool special = (T == rb) || (j_tile < p.bias.sink_len) ||
                           (p.bias.window > 0 && j_tile + 127 > 128 * rb - p.bias.window);
      // the whole S tile of this row into registers, then the buffer goes back to the MMA warp at
      // once, so the next tile's QK^T overlaps this tile's exponentials
      float v[4][32];
      {
        uint32_t raw[4][32];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) tmem_ld32(tbase + lane_addr + 128 * w + 32 * cc, raw[cc]);
        tmem_wait_ld();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
          for (int t = 0; t < 32; ++t) v[cc][t] = __uint_as_float(raw[cc][t]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.s_empty[w]);
      float sum[4] = {0.f, 0.f, 0.f, 0.f};
      // Ordinary tiles once the rows have a reference: the exponentials first, against it.  Their
      // sum bounds their largest term, so a row whose sum is at most 2^kRescale has no logit more
      // than kRescale above the reference, the max pass's own test, and gets that path's results.
      // Otherwise (rare once the reference settles; also an overflow) the max of the shifted
      // values moves the reference of the rows past it, and the exponentials are taken again.
      if (!special && __all_sync(0xffffffffu, c != -INFINITY || !row_ok)) {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const float o = kbo[cc] - c;
#pragma unroll
          for (int t = 0; t < 32; ++t) v[cc][t] = fmaf(v[cc][t], p.a, o);
          sum[cc] = sum_ex2_32(v[cc]);
        }
        const bool big = row_ok && !(((sum[0] + sum[1]) + (sum[2] + sum[3])) <= kRescaleSum);
        if (__any_sync(0xffffffffu, big)) {
          const float m = fmaxf(fmaxf(warp_max32(v[0]), warp_max32(v[1])), fmaxf(warp_max32(v[2]), warp_max32(v[3])));
          const bool need = row_ok && m > kRescale;
          if (__any_sync(0xffffffffu, need)) {
            const float d = need ? m : 0.f;
            const float f = need ? ex2_approx(-d) : 1.f;
            for (int c0 = 0; c0 < used; c0 += 32) {
              uint32_t xs[32];
              tmem_ld32(tbase + lane_addr + xbase + c0, xs);
              tmem_wait_ld();
#pragma unroll
              for (int t = 0; t < 32; ++t) xs[t] = __float_as_uint(__uint_as_float(xs[t]) * f);
              tmem_st32(tbase + lane_addr + xbase + c0, xs);
            }
            tmem_wait_st();
            c += d;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
#pragma unroll
              for (int t = 0; t < 32; ++t) v[cc][t] -= d;
              sum[cc] = sum_ex2_32(v[cc]);
            }
          }
        }
        if (!row_ok) sum[0] = sum[1] = sum[2] = sum[3] = 0.f;
      } else {
        float mc;
        if (!special) {
          // only the key-block term can apply: a constant per 32 keys
          mc = -INFINITY;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) mc = fmaxf(mc, fmaf(warp_max32(v[cc]), p.a, kbo[cc]));
        } else {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const int j0 = j_tile + 32 * cc;
            const float kb = kb_term(p.bias, h, j0);
#pragma unroll
            for (int t = 0; t < 32; ++t) {
              const int j = j0 + t;
              v[cc][t] = (row_ok && j <= i) ? fmaf(v[cc][t], p.a, bias_with_kb(p.bias, i, j, kb) * kLog2e) : -INFINITY;
            }
          }
          mc = fmaxf(fmaxf(warp_max32(v[0]), warp_max32(v[1])), fmaxf(warp_max32(v[2]), warp_max32(v[3])));
        }
        if (!row_ok) mc = -INFINITY;
        const bool need = mc > c + kRescale;
        if (__any_sync(0xffffffffu, need)) {
          const float cn = need ? mc : c;
          const float f = need ? ex2_approx(c - cn) : 1.f;  // c = -inf gives 0
          for (int c0 = 0; c0 < used; c0 += 32) {
            uint32_t xs[32];
            tmem_ld32(tbase + lane_addr + xbase + c0, xs);
            tmem_wait_ld();
#pragma unroll
            for (int t = 0; t < 32; ++t) xs[t] = __float_as_uint(__uint_as_float(xs[t]) * f);
            tmem_st32(tbase + lane_addr + xbase + c0, xs);
          }
          tmem_wait_st();
          c = cn;
        }
        if (c != -INFINITY && row_ok) {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            if (!special) {
              const float o = kbo[cc] - c;
#pragma unroll
              for (int t = 0; t < 32; ++t) v[cc][t] = fmaf(v[cc][t], p.a, o);
            } else {
#pragma unroll
              for (int t = 0; t < 32; ++t) v[cc][t] -= c;  // -inf stays -inf and gives 0
            }
            sum[cc] = sum_ex2_32(v[cc]);
          }
        }
      }
      // block sums of this tile: one 128-key block, or two 64-key blocks
      float acc[2];
      if (p.B == 64) {
        acc[0] = sum[0] + sum[1];
        acc[1] = sum[2] + sum[3];
      } else {
        acc[0] = (sum[0] + sum[1]) + (sum[2] + sum[3]);
        acc[1] = 0.f;
      }
      if (per_tile == 1)
        tmem_st1(tbase + lane_addr + xbase + used, __float_as_uint(acc[0]));
      else
        tmem_st2(tbase + lane_addr + xbase + used, __float_as_uint(acc[0]), __float_as_uint(acc[1]));
      used += per_tile;
    }
    tmem_wait_st();

    // ---- merge the two warpgroups' references and sums into the row normaliser ----
    float l = 0.f;
    for (int c0 = 0; c0 < used; c0 += 32) {
      uint32_t xs[32];
      tmem_ld32(tbase + lane_addr + xbase + c0, xs);
      tmem_wait_ld();
#pragma unroll
      for (int t = 0; t < 32; ++t)
        if (c0 + t < used) l += __uint_as_float(xs[t]);
    }
    s.cref[w][row] = c;
    s.csum[w][row] = l;
    named_sync(1, 256);
    // both warpgroups have left their tile loops: the failure flag is stable until the next unit
    const bool good = s.sm_fail == 0;
    const float co = s.cref[1 - w][row], lo = s.csum[1 - w][row];
    const float C = fmaxf(c, co);
    float Ls = 0.f;
    if (C != -INFINITY) {
      if (c != -INFINITY) Ls += l * ex2_approx(c - C);
      if (co != -INFINITY) Ls += lo * ex2_approx(co - C);
    }
    const float lse2 = C + __log2f(Ls);
    if (w == 0 && row_ok && good && checked(p.ws, h < p.H && i < p.L, 0xC11)) {
      const size_t gi = (size_t)h * p.L + i;
      p.lse_ws[gi] = lse2 * kLn2;
      if (p.lse_out) p.lse_out[gi] = lse2 * kLn2;
    }
    const float scale = (row_ok && Ls > 0.f && c != -INFINITY) ? ex2_approx(c - C) / Ls : 0.f;

    // ---- normalised block sums, reduced over this warp's 32 rows ----
    for (int c0 = 0; c0 < used; c0 += 32) {
      uint32_t xs[32];
      tmem_ld32(tbase + lane_addr + xbase + c0, xs);
      tmem_wait_ld();
      float v[32];
#pragma unroll
      for (int t = 0; t < 32; ++t) v[t] = __uint_as_float(xs[t]) * scale;
      // sum each of the 32 columns over the warp's 32 rows: every step hands half of the columns
      // still held to the partner lane and adds the other half, so after five steps lane l holds
      // the sum of column l (31 shuffles instead of 5 per column)
#pragma unroll
      for (int o = 16, n = 32; o >= 1; o >>= 1, n >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int t = 0; t < n / 2; ++t) {
          const float send = upper ? v[t] : v[t + n / 2];
          const float keep = upper ? v[t + n / 2] : v[t];
          v[t] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      if (c0 + lane < used) s.red[w][q4][c0 + lane] = v[0];
    }
    named_sync(1, 256);
    // block masses: own columns -> key blocks
    const int nblk = (p.B == 128) ? 1 : 2;
    for (int col = gtid; col < used; col += 128) {
      int jb;
      if (p.B == 128) {
        jb = 2 * col + w;
        s.mass[0][jb] = (s.red[w][0][col] + s.red[w][1][col] + s.red[w][2][col] + s.red[w][3][col]) * (1.f / 128.f);
      } else {
        jb = 4 * (col >> 1) + 2 * w + (col & 1);
        s.mass[0][jb] = (s.red[w][0][col] + s.red[w][1][col]) * (1.f / 64.f);
        s.mass[1][jb] = (s.red[w][2][col] + s.red[w][3][col]) * (1.f / 64.f);
      }
    }
    named_sync(1, 256);

    // ---- selection: warpgroup w selects query block w of the unit ----
    const int I = (p.B == 128) ? rb : 2 * rb + w;
    const bool sel = (w < nblk) && I < p.nqb && I >= p.qb0 && I < p.qb1 && good;
    const uint32_t bar_id = 2 + w;
    if (sel) {
      const int n = I + 1;
      float* m = s.mass[w];
      for (int J = gtid; J < n; J += 128) {
        const uint64_t kj = ((uint64_t)__float_as_uint(m[J]) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)J);
        int rank = 0;
        for (int t = 0; t < n; ++t) {
          const uint64_t kt = ((uint64_t)__float_as_uint(m[t]) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)t);
          rank += (kt > kj);
        }
        s.sorted[w][rank] = J;
      }
      if (gtid < 8) s.bits[w][gtid] = 0u;
      named_sync(bar_id, 128);
      if (gtid < 32) {
        // fp64 prefix sum of the sorted masses: lane holds entries 8*lane .. 8*lane + 7
        double loc[8];
        double tot = 0.0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int idx = 8 * gtid + e;
          loc[e] = idx < n ? (double)m[s.sorted[w][idx]] : 0.0;
          tot += loc[e];
        }
        double incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const double y = __shfl_up_sync(0xffffffffu, incl, o);
          if (gtid >= o) incl += y;
        }
        double run = incl - tot;
        int first = 1 << 30;
        double at = 0.0;
        const double pd = (double)p.p;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int idx = 8 * gtid + e;
          run += loc[e];
          if (idx < n && first == (1 << 30) && run >= pd) {
            first = idx;
            at = run;
          }
        }
        const uint32_t hit = __ballot_sync(0xffffffffu, first != (1 << 30));
        int kstar;
        double km;
        if (p.p >= 1.f || hit == 0u) {
          kstar = n;
          km = __shfl_sync(0xffffffffu, incl, 31);
        } else {
          const int src = __ffs(hit) - 1;
          kstar = __shfl_sync(0xffffffffu, first, src) + 1;
          km = __shfl_sync(0xffffffffu, at, src);
        }
        if (gtid == 0) {
          s.kstar[w] = kstar;
          s.kmass[w] = (float)km;
        }
      }
      named_sync(bar_id, 128);
      const int kstar = s.kstar[w];
      for (int t = gtid; t < kstar; t += 128) atomicOr(&s.bits[w][s.sorted[w][t] >> 5], 1u << (s.sorted[w][t] & 31));
      named_sync(bar_id, 128);
      const int u = h * p.nqb + I;
      if (checked(p.ws, h < p.H && I >= 0 && I < p.nqb, 0xC12)) {
        if (gtid < p.nkw) p.kept_bits[(size_t)u * p.nkw + gtid] = s.bits[w][gtid];
        if (gtid == 0) {
          p.count_ws[u] = kstar;
          p.kept_mass[u] = s.kmass[w];
        }
        if (p.mass_out)
          for (int J = gtid; J < p.nqb; J += 128) p.mass_out[(size_t)u * p.nqb + J] = J <= I ? m[J] : 0.f;
      }
    }
    named_sync(1, 256);  // the shared arrays are reused by the next unit
    if (p.renorm) {
      // kept mass of this thread's row: its normalised block sums of the kept blocks of the row's
      // query block, over both warpgroups' columns; the emit's normaliser then absorbs it
      const int qrow = (p.B == 128) ? 0 : (row >> 6);
      const int Irow = (p.B == 128) ? rb : 2 * rb + qrow;
      float part = 0.f;
      for (int c0 = 0; c0 < used; c0 += 32) {
        uint32_t xs[32];
        tmem_ld32(tbase + lane_addr + xbase + c0, xs);
        tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const int col = c0 + t;
          const int J = (p.B == 128) ? 2 * col + w : 4 * (col >> 1) + 2 * w + (col & 1);
          if (col < used && J <= Irow && ((s.bits[qrow][J >> 5] >> (J & 31)) & 1u)) part += __uint_as_float(xs[t]);
        }
      }
      s.csum[w][row] = part * scale;
      named_sync(1, 256);
      if (w == 0 && row_ok && good && Irow >= p.qb0 && Irow < p.qb1) {
        const float m = s.csum[0][row] + s.csum[1][row];
        if (m > 0.f) p.lse_ws[(size_t)h * p.L + i] += logf(m);
      }
    }
    const bool stop = s.sm_fail != 0;
    named_sync(1, 256);  // nobody starts the next unit's tiles before everyone has read the flag
    if (stop) break;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    k_compress_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk, Params p) {
  extern __shared__ unsigned char smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&s.q_full, 1);
    mbar_init(&s.q_empty, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&s.k_full[i], 1);
      mbar_init(&s.k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.s_empty[i], 4);
    }
    mbar_init(&s.mma_done, 1);
    s.abort = 0;
    s.sm_fail = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&s.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp < kSoftmaxWarp0) {
    regs_dec<kRegsControl>();
    if (warp == kProducerWarp)
      producer(s, p, &tq, &tk);
    else if (warp == kMmaWarp)
      mma_issuer(s, p);
  } else {
    regs_inc<kRegsSoftmax>();
    softmax_group(s, p, (warp - kSoftmaxWarp0) >> 2);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(s.tmem_base, 512);
}

}  // namespace

bool tc_compress_supported(const CompressArgs& a) {
  return a.dt == MR_BF16 && a.d == 128 && (a.block == 64 || a.block == 128) && a.scale > 0.f &&
         (a.bias.kb == nullptr || a.bias.kb_block % 32 == 0);
}

cudaError_t tc_compress_stats(const CompressArgs& a) {
  Params p;
  p.H = a.H;
  p.L = a.L;
  p.B = a.block;
  p.nqb = a.L / a.block;
  p.nkw = (p.nqb + 31) / 32;
  // 128-row blocks holding the query blocks qb0 .. qb1 - 1
  const int rb_lo = a.block == 128 ? a.qb0 : a.qb0 / 2;
  p.rb_hi = a.block == 128 ? a.qb1 : (a.qb1 + 1) / 2;
  p.n_rb = p.rb_hi - rb_lo;
  p.n_units = p.H * p.n_rb;
  p.qb0 = a.qb0;
  p.qb1 = a.qb1;
  p.renorm = a.map.renormalised != 0;
  p.a = a.scale * kLog2e;
  p.p = a.p;
  p.bias = a.bias;
  p.lse_ws = a.lse_ws;
  p.count_ws = a.count_ws;
  p.kept_bits = a.map.kept_bits;
  p.kept_mass = a.map.kept_mass;
  p.mass_out = a.map.mass;
  p.lse_out = a.map.lse;
  p.ws = a.ws;
  CUtensorMap tq, tk;
  const uint64_t rows = (uint64_t)a.H * a.L;
  if (!make_tmap_bf16_2d(&tq, a.Q, 128, rows, 256, 64, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tk, a.K, 128, rows, 256, 64, 128)) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = p.n_units < sms ? p.n_units : sms;
  // the register split assumes the launch allocation it was sized for
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, k_compress_tc);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  const size_t smem = sizeof(Smem) + 1024;
  e = cudaFuncSetAttribute(k_compress_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps(kKCompressTc, a.stream);
  k_compress_tc<<<grid, kThreads, smem, a.stream>>>(tq, tk, p);
  return cudaGetLastError();
}

}  // namespace mr
