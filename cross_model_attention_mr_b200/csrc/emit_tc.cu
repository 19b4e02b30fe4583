// Emit the kept tiles of the compressed map on sm_100a (bf16 Q/K, d = 128): MapFlow section 5.2,
// "stores retained attention blocks in BSR format".
//
// After the statistics pass and the scan of kept counts, every kept tile (h, I, J) is recomputed:
// S = Q_I K_J^T on the tensor core, P_ij = 2^(s'_ij - lse2_i) (s' the biased logit in base 2,
// lse2 the row log-normaliser; zero above the causal diagonal), rounded to bf16 and written in
// the map's storage order (128-byte swizzled panels) to its BSR position.  Tiles that no query
// block of the unit kept are neither loaded nor multiplied.  Each tile leaves shared memory with
// one bulk store, so the pass is bound by the HBM write of the map.
//
// Roles per CTA (persistent, units longest-first): TMA producer warp (Q rows, ring of needed K
// tiles), MMA warp (128 x 128 tiles into two Tensor Memory buffers), two warpgroups that take
// alternate needed tiles (one query row per thread).  All waits are bounded.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"
#include "profile.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace mr {
namespace {

using namespace sm100;

// Warpgroup 0: TMA producer warp, MMA warp, two idle warps; warpgroups 1..kWG: emitting
// warpgroups, which take the unit's needed tiles in turn.  Three of them put three emitting warps
// on every SM sub-partition (the kernel is bound by their latency); warpgroup 0 drops to 56
// registers so they can rise to 152 each: 56 + 3 x 152 = 4 x 128, the launch allocation.
constexpr int kWG = 3;
constexpr int kThreads = 128 * (kWG + 1);
constexpr int kLaunchRegs = 128;
constexpr int kRegsControl = 56;
constexpr int kRegsEmit = 152;
static_assert(kRegsControl + kWG * kRegsEmit == (kWG + 1) * kLaunchRegs, "register split");
constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kSoftmaxWarp0 = 4;
constexpr int kKStages = 3;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLog2Fp8Max = 8.807354922057604f;  // log2(448), 448 = largest e4m3 value

struct Params {
  int H, L, B, nqb, nkw, n_rb, n_units;
  int rb_hi;  // units cover 128-row blocks rb_hi - n_rb .. rb_hi - 1
  float a;
  Bias bias;
  const float* lse_ws;
  const int32_t* row_ptr;
  const uint32_t* kept_bits;
  int64_t capacity;
  int32_t* col_idx;
  __nv_bfloat16* vals;   // bf16 maps
  uint8_t* vals8;        // fp8 (e4m3) maps
  float* tile_scale;     // fp8 maps: one scale per 32-row x 64-key piece
  WsHeader* ws;
};

struct Smem {
  __nv_bfloat16 q[2][128 * 64];
  __nv_bfloat16 k[kKStages][2][128 * 64];
  __nv_bfloat16 stage[kWG][128 * 128];  // per warpgroup: 4 warps x (2 key halves x 32 rows x 128 B)
  uint64_t q_full, q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t s_full[kWG], s_empty[kWG];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};

static_assert(sizeof(Smem) + 1024 <= 232448, "shared memory (plus alignment slack) must fit the 227 KB opt-in limit");

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

// One query block's kept bits, walked with non-decreasing J: kept flag, and the BSR position of
// each kept tile (row start + kept blocks so far).
struct QCursor {
  const uint32_t* bits;
  uint32_t word;
  int word_idx, count, I;
  int64_t first;
  bool live;
  __device__ __forceinline__ void start(const Params& p, int h, int I_) {
    I = I_;
    live = I_ >= 0 && I_ < p.nqb;
    count = 0;
    word_idx = 0;
    word = 0u;
    first = 0;
    bits = nullptr;
    if (live) {
      const int u = h * p.nqb + I_;
      bits = p.kept_bits + (size_t)u * p.nkw;
      word = __ldg(bits);
      first = __ldg(p.row_ptr + u);
    }
  }
  __device__ __forceinline__ bool kept(int J) {
    if (!live || J > I) return false;
    const int wi = J >> 5;
    if (wi != word_idx) {
      word_idx = wi;
      word = __ldg(bits + wi);
    }
    return (word >> (J & 31)) & 1u;
  }
};

// The unit's one (block 128) or two (block 64) query blocks.  pieces(T) returns which pieces of
// key tile T are stored -- bit (2 * row half + key half) for block 64, bit 0 for block 128 -- with
// their BSR positions, and must be called for every T in increasing order.
struct UnitCursor {
  QCursor q[2];
  __device__ __forceinline__ void start(const Params& p, int h, int rb) {
    if (p.B == 128) {
      q[0].start(p, h, rb);
      q[1].start(p, h, -1);
    } else {
      q[0].start(p, h, 2 * rb);
      q[1].start(p, h, 2 * rb + 1);
    }
  }
  __device__ __forceinline__ uint32_t pieces(const Params& p, int T, int64_t (&t)[4]) {
    uint32_t m = 0;
    if (p.B == 128) {
      if (q[0].kept(T)) {
        m = 1u;
        t[0] = q[0].first + q[0].count++;
      }
      return m;
    }
#pragma unroll
    for (int rh = 0; rh < 2; ++rh)
#pragma unroll
      for (int ch = 0; ch < 2; ++ch)
        if (q[rh].kept(2 * T + ch)) {
          m |= 1u << (2 * rh + ch);
          t[2 * rh + ch] = q[rh].first + q[rh].count++;
        }
    return m;
  }
};

__device__ void producer(Smem& s, const Params& p, const CUtensorMap* tq, const CUtensorMap* tk) {
  if ((threadIdx.x & 31) != 0) return;
  uint32_t nk = 0, nu = 0;
  bool ok = true;
  for (int k = blockIdx.x; k < p.n_units && ok; k += gridDim.x, ++nu) {
    int h, rb;
    unit_of(p, k, h, rb);
    if (nu > 0 && !mbar_wait(&s.q_empty, (nu - 1) & 1, &s.abort, kTimeoutNs)) {
      fail(s, p, 0x501);
      break;
    }
    const int qrow = h * p.L + 128 * rb;
    mbar_arrive_expect_tx(&s.q_full, 2 * 128 * 64 * 2);
    tma_load_2d(&s.q[0][0], tq, &s.q_full, 0, qrow);
    tma_load_2d(&s.q[1][0], tq, &s.q_full, 64, qrow);
    UnitCursor uc;
    uc.start(p, h, rb);
    for (int T = 0; T <= rb; ++T) {
      int64_t tpos[4];
      if (!uc.pieces(p, T, tpos)) continue;
      const int st = (int)(nk % kKStages);
      if (nk >= (uint32_t)kKStages && !mbar_wait(&s.k_empty[st], ((nk / kKStages) - 1) & 1, &s.abort, kTimeoutNs)) {
        fail(s, p, 0x502);
        ok = false;
        break;
      }
      const int krow = h * p.L + 128 * T;
      mbar_arrive_expect_tx(&s.k_full[st], 2 * 128 * 64 * 2);
      tma_load_2d(&s.k[st][0][0], tk, &s.k_full[st], 0, krow);
      tma_load_2d(&s.k[st][1][0], tk, &s.k_full[st], 64, krow);
      ++nk;
    }
  }
  const int never = 0;
  for (uint32_t g = (nk > (uint32_t)kKStages ? nk - kKStages : 0); g < nk; ++g)
    mbar_wait(&s.k_full[g % kKStages], (g / kKStages) & 1, &never, kTimeoutNs);
  if (nu > 0) mbar_wait(&s.q_full, (nu - 1) & 1, &never, kTimeoutNs);
}

__device__ void mma_issuer(Smem& s, const Params& p) {
  if ((threadIdx.x & 31) != 0) return;
  const uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
  const uint32_t tbase = s.tmem_base;
  uint32_t nk = 0, nu = 0, nb[kWG] = {};
  bool ok = true;
  for (int k = blockIdx.x; k < p.n_units && ok; k += gridDim.x, ++nu) {
    int h, rb;
    unit_of(p, k, h, rb);
    if (!mbar_wait(&s.q_full, nu & 1, &s.abort, kTimeoutNs)) {
      fail(s, p, 0x511);
      break;
    }
    int n_local = 0;
    UnitCursor uc;
    uc.start(p, h, rb);
    for (int T = 0; T <= rb; ++T) {
      int64_t tpos[4];
      if (!uc.pieces(p, T, tpos)) continue;
      const int st = (int)(nk % kKStages), b = n_local % kWG;
      if (!mbar_wait(&s.k_full[st], (nk / kKStages) & 1, &s.abort, kTimeoutNs) ||
          (nb[b] > 0 && !mbar_wait(&s.s_empty[b], (nb[b] - 1) & 1, &s.abort, kTimeoutNs))) {
        fail(s, p, 0x512);
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
      ++nk;
      ++n_local;
    }
    if (ok) mma_commit(&s.q_empty);
  }
  mma_commit(&s.mma_done);
  const int never = 0;
  mbar_wait(&s.mma_done, 0, &never, kTimeoutNs);
}

__device__ __forceinline__ float kb_offset(const Bias& b, int h, int j) {
  if (b.kb == nullptr) return 0.f;
  const float v = __ldg(b.kb + (size_t)h * b.n_kb + j / b.kb_block);
  return v == -INFINITY ? 0.f : v * kLog2e;
}

// One warpgroup: each warp handles 32 query rows of every tile given to the warpgroup, stages
// them in the map's storage order and stores them with its own bulk copies (the 32 rows of a
// panel are contiguous in the stored tile), so the warps of the group never wait on each other.
template <bool F8>
__device__ void emit_group(Smem& s, const Params& p, int w) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q4 = warp & 3;
  const int row = 32 * q4 + lane;
  const uint32_t tbase = s.tmem_base;
  const uint32_t lane_addr = (uint32_t)(32 * q4) << 16;
  char* stage = reinterpret_cast<char*>(&s.stage[w][0]) + 8192 * q4;  // 2 x 4 KB: key halves
  const int rh = row >> 6;  // block 64: which query block of the unit this warp's rows belong to
  uint32_t nb = 0;
  bool store_pending = false;
  bool ok = true;
  for (int k = blockIdx.x; k < p.n_units && ok; k += gridDim.x) {
    int h, rb;
    unit_of(p, k, h, rb);
    const int i = 128 * rb + row;
    const bool row_ok = i < p.L;
    const float lse2 = row_ok ? __ldg(p.lse_ws + (size_t)h * p.L + i) * kLog2e : 0.f;
    UnitCursor uc;
    uc.start(p, h, rb);
    int n_local = 0;
    for (int T = 0; T <= rb; ++T) {
      int64_t tpos[4];
      const uint32_t pieces = uc.pieces(p, T, tpos);
      if (!pieces) continue;
      const int mine = n_local++ % kWG;
      if (mine != w) continue;
      if (!mbar_wait(&s.s_full[w], nb & 1, &s.abort, kTimeoutNs)) {
        fail(s, p, 0x521);
        ok = false;
        break;
      }
      ++nb;
      tc_fence_after();
      // the staging buffer may still be read by this warp's previous bulk stores
      if (store_pending) {
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
      }
      const int j_tile = 128 * T;
      const bool special = (T == rb) || (j_tile < p.bias.sink_len) ||
                           (p.bias.window > 0 && j_tile + 127 > 128 * rb - p.bias.window);
      // which 64-key halves of this warp's rows are stored
      const uint32_t row_mask = p.B == 128 ? 3u : ((pieces >> (2 * rh)) & 3u);
      float sc[2] = {0.f, 0.f};  // fp8: scale of each stored piece
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t raw[2][32];
        tmem_ld32(tbase + lane_addr + 128 * w + 64 * hh, raw[0]);
        tmem_ld32(tbase + lane_addr + 128 * w + 64 * hh + 32, raw[1]);
        tmem_wait_ld();
        if (hh == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s.s_empty[w]);
        }
        if (!((row_mask >> hh) & 1u)) continue;  // warp-uniform
        if (F8 && !special) {
          // fp8, bias constant per 32 keys: the piece maximum comes from the raw logits (a > 0),
          // so each value is produced already scaled, P * 448 / max = 2^(x + log2 448 - max x),
          // by one FMA and one exponential
          float ob[2], mxl = -INFINITY;
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            ob[cc] = kb_offset(p.bias, h, j_tile + 64 * hh + 32 * cc) - lse2;
            float m = __uint_as_float(raw[cc][0]);
#pragma unroll
            for (int t = 1; t < 32; ++t) m = fmaxf(m, __uint_as_float(raw[cc][t]));
            mxl = fmaxf(mxl, fmaf(m, p.a, ob[cc]));
          }
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) mxl = fmaxf(mxl, __shfl_xor_sync(0xffffffffu, mxl, o));
          sc[hh] = ex2_approx(mxl) / kFp8Max;
          const float shift = kLog2Fp8Max - mxl;
          char* dst = stage + 2048 * hh + lane * 64;
#pragma unroll
          for (int c16 = 0; c16 < 4; ++c16) {
            const int cc = c16 >> 1;
            const float o = ob[cc] + shift;
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int x = 16 * (c16 & 1) + 4 * e;
              float q[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) q[u] = ex2_approx(fmaf(__uint_as_float(raw[cc][x + u]), p.a, o));
              const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(q[0], q[1]), __NV_SATFINITE, __NV_E4M3);
              const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(q[2], q[3]), __NV_SATFINITE, __NV_E4M3);
              pk[e] = __byte_perm(lo, hi, 0x5140);  // bytes of keys (0, 2, 1, 3)
            }
            *reinterpret_cast<uint4*>(dst + 16 * c16) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
          continue;
        }
        float pr[64];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int j0 = j_tile + 64 * hh + 32 * cc;
          if (!special) {
            const float o = kb_offset(p.bias, h, j0) - lse2;
#pragma unroll
            for (int t = 0; t < 32; ++t) pr[32 * cc + t] = ex2_approx(fmaf(__uint_as_float(raw[cc][t]), p.a, o));
          } else {
            const float kb = kb_term(p.bias, h, j0);
#pragma unroll
            for (int t = 0; t < 32; ++t) {
              const int j = j0 + t;
              pr[32 * cc + t] = (row_ok && j <= i)
                                    ? ex2_approx(fmaf(__uint_as_float(raw[cc][t]), p.a, bias_with_kb(p.bias, i, j, kb) * kLog2e) - lse2)
                                    : 0.f;
            }
          }
        }
        if (!F8) {
          char* dst = stage + 4096 * hh + lane * 128;
#pragma unroll
          for (int c8 = 0; c8 < 8; ++c8) {  // 16-byte chunk of the 64-column panel row, swizzled
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 b2 = __floats2bfloat162_rn(pr[8 * c8 + 2 * e], pr[8 * c8 + 2 * e + 1]);
              pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            *reinterpret_cast<uint4*>(dst + ((c8 ^ (lane & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        } else {
          // the warp's 32 rows x 64 keys are one piece: scale = max / 448, values stored as e4m3
          float mx = 0.f;
#pragma unroll
          for (int t = 0; t < 64; ++t) mx = fmaxf(mx, pr[t]);
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          sc[hh] = mx / kFp8Max;
          const float inv = mx > 0.f ? kFp8Max / mx : 0.f;
          char* dst = stage + 2048 * hh + lane * 64;
#pragma unroll
          for (int c16 = 0; c16 < 4; ++c16) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int x = 16 * c16 + 4 * e;
              const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(pr[x] * inv, pr[x + 1] * inv), __NV_SATFINITE, __NV_E4M3);
              const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(pr[x + 2] * inv, pr[x + 3] * inv), __NV_SATFINITE, __NV_E4M3);
              pk[e] = __byte_perm(lo, hi, 0x5140);  // bytes of keys (0, 2, 1, 3)
            }
            *reinterpret_cast<uint4*>(dst + 16 * c16) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        bool issued = false;
        for (int hh = 0; hh < 2; ++hh) {
          if (!((row_mask >> hh) & 1u)) continue;
          const int piece = p.B == 128 ? 0 : 2 * rh + hh;
          const int64_t t = tpos[piece];
          if (t >= p.capacity) continue;
          if (!checked(p.ws, t >= 0 && (p.B == 128 ? T : 2 * T + hh) < p.nqb, 0xC21)) continue;
          // destination: panel hh of the 128-tile, or the (rh, hh) 64-tile; this warp's 32 rows
          if (!F8) {
            const int64_t tbytes = (int64_t)p.B * p.B * 2;
            char* gdst = reinterpret_cast<char*>(p.vals) + t * tbytes +
                         (p.B == 128 ? 16384 * hh + 4096 * q4 : 4096 * (q4 & 1));
            bulk_s2g(gdst, stage + 4096 * hh, 4096);
          } else {
            const int64_t tbytes = (int64_t)p.B * p.B;
            char* gdst = reinterpret_cast<char*>(p.vals8) + t * tbytes +
                         (p.B == 128 ? 8192 * hh + 2048 * q4 : 2048 * (q4 & 1));
            bulk_s2g(gdst, stage + 2048 * hh, 2048);
            const int rg = p.B == 128 ? q4 : (q4 & 1);
            p.tile_scale[t * fp8_scales_per_tile(p.B) + rg * (p.B / 64) + (p.B == 128 ? hh : 0)] = sc[hh];
          }
          issued = true;
          const bool writer = p.B == 128 ? (q4 == 0 && hh == 0) : ((q4 & 1) == 0);
          if (writer) p.col_idx[t] = p.B == 128 ? T : 2 * T + hh;
        }
        if (issued) {
          bulk_commit();
          store_pending = true;
        }
      }
      store_pending = __shfl_sync(0xffffffffu, store_pending ? 1 : 0, 0) != 0;
    }
  }
  if (lane == 0 && store_pending) bulk_wait_all<0>();
  __syncwarp();
}

template <bool F8>
__global__ void __launch_bounds__(kThreads, 1)
    k_emit_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk, Params p) {
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
    for (int i = 0; i < kWG; ++i) {
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.s_empty[i], 4);
    }
    mbar_init(&s.mma_done, 1);
    s.abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&s.tmem_base, 512);  // kWG S buffers of 128 columns (allocations are powers of two)
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // every warp of warpgroup 0 gives its registers back before any role starts: the emitting
  // warpgroups' increase waits for them
  if (warp < kSoftmaxWarp0) {
    regs_dec<kRegsControl>();
    if (warp == kProducerWarp)
      producer(s, p, &tq, &tk);
    else if (warp == kMmaWarp)
      mma_issuer(s, p);
  } else {
    regs_inc<kRegsEmit>();
    emit_group<F8>(s, p, (warp - kSoftmaxWarp0) >> 2);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(s.tmem_base, 512);
}

}  // namespace

cudaError_t tc_emit(const CompressArgs& a) {
  Params p;
  p.H = a.H;
  p.L = a.L;
  p.B = a.block;
  p.nqb = a.L / a.block;
  p.nkw = (p.nqb + 31) / 32;
  // rows of query blocks outside qb0 .. qb1 - 1 keep no tiles (their counts are 0)
  const int rb_lo = a.block == 128 ? a.qb0 : a.qb0 / 2;
  p.rb_hi = a.block == 128 ? a.qb1 : (a.qb1 + 1) / 2;
  p.n_rb = p.rb_hi - rb_lo;
  p.n_units = p.H * p.n_rb;
  p.a = a.scale * kLog2e;
  p.bias = a.bias;
  p.lse_ws = a.lse_ws;
  p.row_ptr = a.map.row_ptr;
  p.kept_bits = a.map.kept_bits;
  p.capacity = a.map.capacity_tiles;
  p.col_idx = a.map.col_idx;
  p.vals = (__nv_bfloat16*)a.map.vals;
  p.vals8 = (uint8_t*)a.map.vals;
  p.tile_scale = a.map.tile_scale;
  p.ws = a.ws;
  CUtensorMap tq, tk;
  const uint64_t rows = (uint64_t)a.H * a.L;
  if (!make_tmap_bf16_2d(&tq, a.Q, 128, rows, 256, 64, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16_2d(&tk, a.K, 128, rows, 256, 64, 128)) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = p.n_units < sms ? p.n_units : sms;
  const size_t smem = sizeof(Smem) + 1024;
  const bool f8 = a.map.val_dtype == MR_FP8_E4M3;
  auto kern = f8 ? k_emit_tc<true> : k_emit_tc<false>;
  // the register split assumes the launch allocation it was sized for; anything else could leave
  // an increase waiting for registers that do not exist
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps(kKEmitTc, a.stream);
  kern<<<grid, kThreads, smem, a.stream>>>(tq, tk, p);
  return cudaGetLastError();
}

}  // namespace mr
