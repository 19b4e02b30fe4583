// Exact causal attention on sm_100a (bf16, d = d_v = 128): O = softmax(s) V with
// s_ij = scale * q_i.k_j + b(h, i, j) over keys j <= i ("AttnCache Guide", "The Quadratic
// Self-Attention Cost"), for packed variable-length sequences with a query offset (MapFlow
// section 6, variable-length packing).  It is the reference the method is compared against and
// the path for the rows a receiver does not reuse.
//
// One CTA per (head, pair of consecutive 128-row query tiles A and B of one sequence), the pairs
// holding the most keys first.  Tensor Memory holds S and O of both tiles (4 x 128 columns).
//   * producer warp: TMA loads of both Q tiles, then the 128-key K and V tiles in the order the
//     MMA warp consumes them (K_0, K_1, V_0, K_2, V_1, ...) through a 3-slot ring (128-byte
//     swizzle); a slot is released when every MMA that reads it has completed;
//   * MMA warp: for each key tile j, S_A = Q_A K_j^T and S_B = Q_B K_j^T, then, one key tile
//     behind, O_A += P_A V_{j-1} and O_B += P_B V_{j-1} (P from shared memory, V MN-major), so
//     each softmax warpgroup's exponentials run while the tensor core works on the other tile;
//   * two softmax warpgroups, one per tile, a query row per thread: read S, apply the causal mask
//     and the logit bias, keep a row reference that moves only when a logit exceeds it by more than
//     2^8 (the tile's O is then rescaled in Tensor Memory), and write P = 2^(s' - reference) as a
//     bf16 128-byte-swizzled operand; at the end divide O by the row sum and store it.
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

// Warpgroup 0: producer warp, MMA warp, two idle warps; warpgroups 1 and 2: softmax of tiles A
// and B (warp w reads Tensor Memory lanes 32 (w % 4) ..).  Each SM sub-partition holds one warp of
// each warpgroup, so the register split 72 + 216 + 216 uses exactly the launch's 3 x 168.
constexpr int kThreads = 384;
constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kSoftmaxWarp0 = 4;
constexpr int kLaunchRegs = 168;
constexpr int kRegsControl = 72;
constexpr int kRegsSoftmax = 216;
static_assert(kRegsControl + 2 * kRegsSoftmax == 3 * kLaunchRegs, "register split");
constexpr int kSlots = 3;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescale = 8.0f;
constexpr uint32_t kTileBytes = 128 * 128 * 2;
// which of every 8 pairs of probabilities take the FMA-pipe exponential (bit k: pair 8 m + k); the
// rest go to the multi-function unit, whose 16 results per clock per SM otherwise bound the softmax
// (measured: 1 pair in 8 beats 2 and 0)
constexpr uint32_t kEmuMask = 0x80;

struct Params {
  const int32_t* cu_q;
  const int32_t* cu_k;
  const int32_t* q_offset;
  int n_seq, H, total_q, total_k;
  float a;  // scale * log2(e)
  Bias bias;
  __nv_bfloat16* O;
  WsHeader* ws;
  uint64_t wait_ns;  // limit of the producer's and MMA warp's protocol waits (drains keep kTimeoutNs);
                     // the softmax warpgroups, furthest downstream, wait twice as long, so the wait
                     // nearest a stall is the one that reports it
  int skip_arrive;   // failure-path test: tile A's softmax withholds its first "P ready" arrive
};

struct Smem {
  __nv_bfloat16 q[2][2][128 * 64];        // [tile][d half][row][64]
  __nv_bfloat16 kv[kSlots][2][128 * 64];  // [slot][column half][key][64]
  __nv_bfloat16 p[2][2][128 * 64];        // [tile][key half][row][64]
  uint64_t q_full;
  uint64_t slot_full[kSlots], slot_empty[kSlots];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[2], p_empty[2];
  uint64_t o_full[2], mma_done;
  uint32_t tmem_base;
  int abort;
};

// A CTA's work: query tiles t[0] (A) and t[1] (B; -1 when the pair has one tile) of one sequence.
struct Pair {
  int t[2];
  int q0, len_q;  // first packed query row of the sequence, its query rows
  int k0;         // first packed key row of the sequence
  int off;        // absolute position of the sequence's first query row
  int nk[2];      // key tiles each tile needs (0 for a missing tile B)
};

__device__ __forceinline__ int key_tiles(int off, int t, int len_q) {
  return (off + min(t * 128 + 127, len_q - 1)) / 128 + 1;
}

// The k-th pair in the launch order: the last two tiles of every sequence, then the two before,
// and so on (the pairs with the most keys first); a sequence with an odd tile count ends with a
// one-tile pair at its start.  false when k is past the last pair.
__device__ bool find_pair(const Params& p, int k, Pair& pr) {
  for (int r = 0;; ++r) {
    bool any = false;
    for (int s = 0; s < p.n_seq; ++s) {
      const int lq = __ldg(p.cu_q + s + 1) - __ldg(p.cu_q + s);
      const int nt = (lq + 127) / 128;
      if (2 * r >= nt) continue;
      any = true;
      if (k-- == 0) {
        const int hi = nt - 1 - 2 * r, lo = hi - 1;
        pr.t[0] = lo >= 0 ? lo : hi;
        pr.t[1] = lo >= 0 ? hi : -1;
        pr.q0 = __ldg(p.cu_q + s);
        pr.len_q = lq;
        pr.k0 = __ldg(p.cu_k + s);
        pr.off = p.q_offset ? __ldg(p.q_offset + s) : 0;
        pr.nk[0] = key_tiles(pr.off, pr.t[0], lq);
        pr.nk[1] = pr.t[1] >= 0 ? key_tiles(pr.off, pr.t[1], lq) : 0;
        return true;
      }
    }
    if (!any) return false;
  }
}

// Ring positions in consumption order for nk key tiles: K_0, K_1, V_0, K_2, V_1, ..., V_{nk-1}.
__device__ __forceinline__ int k_item(int j) { return j == 0 ? 0 : 2 * j - 1; }
__device__ __forceinline__ int v_item(int j, int nk) { return min(2 * j + 2, 2 * nk - 1); }

__device__ __forceinline__ void fail(Smem& s, const Params& p, uint32_t detail) {
  set_status(p.ws, MR_ERR_TIMEOUT, detail);
  s.abort = 1;
}

// ------------------------------------------------------------------------------------------------
// Ring item i sits in slot i % 3 (use i / 3 of that slot) and overwrites item i - 3, which the MMA
// warp released before it: the releases come in item order.
__device__ void producer(Smem& s, const Params& p, const Pair& pr, int h, const CUtensorMap* tq,
                         const CUtensorMap* tk, const CUtensorMap* tv) {
  if ((threadIdx.x & 31) != 0) return;
  const int ntl = pr.t[1] >= 0 ? 2 : 1;
  mbar_arrive_expect_tx(&s.q_full, ntl * kTileBytes);
  for (int x = 0; x < ntl; ++x) {
    const int qrow = h * p.total_q + pr.q0 + 128 * pr.t[x];
    tma_load_2d(&s.q[x][0][0], tq, &s.q_full, 0, qrow);
    tma_load_2d(&s.q[x][1][0], tq, &s.q_full, 64, qrow);
  }
  const int nk = max(pr.nk[0], pr.nk[1]);
  int i = 0;
  for (; i < 2 * nk; ++i) {
    const int sl = i % kSlots, u = i / kSlots;
    if (u > 0 && !mbar_wait_sleep(&s.slot_empty[sl], (u - 1) & 1, &s.abort, p.wait_ns, 64)) {
      fail(s, p, 0x901);
      break;
    }
    const bool is_v = i > 0 && ((i & 1) == 0 || i == 2 * nk - 1);
    const int j = !is_v ? (i + 1) >> 1 : (i == 2 * nk - 1 ? nk - 1 : (i - 2) >> 1);
    const int krow = h * p.total_k + pr.k0 + 128 * j;
    const CUtensorMap* m = is_v ? tv : tk;
    mbar_arrive_expect_tx(&s.slot_full[sl], kTileBytes);
    tma_load_2d(&s.kv[sl][0][0], m, &s.slot_full[sl], 0, krow);
    tma_load_2d(&s.kv[sl][1][0], m, &s.slot_full[sl], 64, krow);
  }
  // no load may land after the CTA releases its shared memory
  const int never = 0;
  for (int g = i > kSlots ? i - kSlots : 0; g < i; ++g)
    mbar_wait(&s.slot_full[g % kSlots], (g / kSlots) & 1, &never, kTimeoutNs);
  mbar_wait(&s.q_full, 0, &never, kTimeoutNs);
}

// ------------------------------------------------------------------------------------------------
__device__ void mma_issuer(Smem& s, const Params& p, const Pair& pr) {
  if ((threadIdx.x & 31) != 0) return;
  const uint32_t id_qk = idesc_bf16_f32(128, 128, false, false);
  const uint32_t id_pv = idesc_bf16_f32(128, 128, false, true);
  const uint32_t tbase = s.tmem_base;
  const int nk = max(pr.nk[0], pr.nk[1]);
  bool ok = mbar_wait(&s.q_full, 0, &s.abort, p.wait_ns);
  if (!ok) fail(s, p, 0x911);

  // O_A += P_A V_i and O_B += P_B V_i (the tiles that need key tile i), then V_i's slot is free
  auto pv = [&](int i) -> bool {
    const int it = v_item(i, nk), sl = it % kSlots;
    if (!mbar_wait(&s.slot_full[sl], (it / kSlots) & 1, &s.abort, p.wait_ns)) return false;
    const uint32_t va = smem_u32(&s.kv[sl][0][0]);
    for (int x = 0; x < 2; ++x) {
      if (i >= pr.nk[x]) continue;
      if (!mbar_wait(&s.p_full[x], i & 1, &s.abort, p.wait_ns)) return false;
      tc_fence_after();
      const uint32_t pa[2] = {smem_u32(&s.p[x][0][0]), smem_u32(&s.p[x][1][0])};
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t da = sdesc_sw128(pa[kk >> 2] + 32 * (kk & 3), 16, 1024);
        const uint64_t dv = sdesc_sw128(va + 2048 * kk, 128 * 128, 1024);
        mma_bf16_ss(tbase + 256 * x + 128, da, dv, id_pv, (i > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(&s.p_empty[x]);
      if (i == pr.nk[x] - 1) mma_commit(&s.o_full[x]);  // the tile's last P V
    }
    mma_commit(&s.slot_empty[sl]);
    return true;
  };

  for (int j = 0; j < nk && ok; ++j) {
    const int it = k_item(j), sl = it % kSlots;
    if (!mbar_wait(&s.slot_full[sl], (it / kSlots) & 1, &s.abort, p.wait_ns)) {
      fail(s, p, 0x912);
      ok = false;
      break;
    }
    const uint32_t ka[2] = {smem_u32(&s.kv[sl][0][0]), smem_u32(&s.kv[sl][1][0])};
    for (int x = 0; x < 2; ++x) {
      if (j >= pr.nk[x]) continue;
      // the softmax has read S_x of key tile j - 1
      if (j >= 1 && !mbar_wait(&s.s_empty[x], (j - 1) & 1, &s.abort, p.wait_ns)) {
        fail(s, p, 0x915);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t qa[2] = {smem_u32(&s.q[x][0][0]), smem_u32(&s.q[x][1][0])};
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t da = sdesc_sw128(qa[kk >> 2] + 32 * (kk & 3), 16, 1024);
        const uint64_t db = sdesc_sw128(ka[kk >> 2] + 32 * (kk & 3), 16, 1024);
        mma_bf16_ss(tbase + 256 * x, da, db, id_qk, kk > 0 ? 1u : 0u);
      }
      mma_commit(&s.s_full[x]);
    }
    if (!ok) break;
    mma_commit(&s.slot_empty[sl]);  // K_j has been read by every S MMA of this key tile
    // the previous key tile's P V runs while the softmax warpgroups work on this one
    if (j >= 1 && !pv(j - 1)) {
      fail(s, p, 0x913);
      ok = false;
    }
  }
  if (ok && !pv(nk - 1)) fail(s, p, 0x914);
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

// Softmax warpgroup of tile x: S_x at Tensor Memory column 256 x, O_x at 256 x + 128, P_x in p[x].
__device__ void softmax_group(Smem& s, const Params& p, const Pair& pr, int h, int x) {
  const int nkx = pr.nk[x];
  const uint64_t wait_ns = 2 * p.wait_ns;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q4 = warp & 3;
  const int row = 32 * q4 + lane;                 // row of the query tile
  const int qi = 128 * pr.t[x] + row;             // row within the sequence
  const bool row_ok = qi < pr.len_q;
  const int pos = pr.off + qi;                    // absolute position: keys 0 .. pos
  const uint32_t tbase = s.tmem_base;
  const uint32_t lane_addr = (uint32_t)(32 * q4) << 16;
  const uint32_t s_col = 256 * x, o_col = 256 * x + 128;
  const int pos0 = pr.off + 128 * pr.t[x];        // position of the tile's first row
  float ref = -INFINITY;                          // row reference (base 2)
  float l = 0.f;                                  // row sum of 2^(s' - ref)
  for (int j = 0; j < nkx; ++j) {
    if (!mbar_wait(&s.s_full[x], j & 1, &s.abort, wait_ns)) {
      fail(s, p, 0x921);
      return;
    }
    tc_fence_after();
    float v[128];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t raw[32];
      tmem_ld32(tbase + lane_addr + s_col + 32 * c, raw);
      tmem_wait_ld();
#pragma unroll
      for (int t = 0; t < 32; ++t) v[32 * c + t] = __uint_as_float(raw[t]);
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.s_empty[x]);

    // x = a s + b - r0 (base 2; r0 the row reference, 0 before the first one): one FMA per logit.
    // Tiles away from the diagonal, the sink and the window carry a per-32-key bias only; the
    // others are masked and biased per element.  Rows past the sequence get x = -inf throughout.
    const float r0 = ref == -INFINITY ? 0.f : ref;
    const int j0 = 128 * j;
    const bool special = (j0 + 127 > pos0) || (j0 < p.bias.sink_len) ||
                         (p.bias.window > 0 && j0 + 127 > pos0 - p.bias.window);
    float mt = -INFINITY;
    if (!special) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float o = row_ok ? kb_log2(p.bias, h, j0 + 32 * c) - r0 : -INFINITY;
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
          v[32 * c + t] = (row_ok && key <= pos)
                              ? fmaf(v[32 * c + t], p.a, bias_with_kb(p.bias, pos, key, kb) * kLog2e - r0)
                              : -INFINITY;
          mt = fmaxf(mt, v[32 * c + t]);
        }
      }
    }
    // P_{j-1} V_{j-1} must have completed before O_x is rescaled or P_x rewritten (one P buffer
    // per tile): that is phase j - 1 of p_empty[x].  Phase j - 2 was waited for before P_{j-1}
    // was written, and phase j cannot complete before this warpgroup writes P_j.
    bool pv_done = j == 0;
    // the reference moves to the row maximum at the first finite logit and whenever a logit passes
    // it by more than 2^8; the tile's x are then re-based and the sums so far rescaled
    const bool need = ref == -INFINITY ? mt > -INFINITY : mt > kRescale;
    if (__any_sync(0xffffffffu, need)) {
      const float f = !need ? 1.f : (ref == -INFINITY ? 0.f : ex2_approx(-mt));
      if (j > 0) {
        if (!mbar_wait(&s.p_empty[x], (j - 1) & 1, &s.abort, wait_ns)) {
          fail(s, p, 0x922);
          return;
        }
        pv_done = true;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t xs[32];
          tmem_ld32(tbase + lane_addr + o_col + 32 * c, xs);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) xs[t] = __float_as_uint(__uint_as_float(xs[t]) * f);
          tmem_st32(tbase + lane_addr + o_col + 32 * c, xs);
        }
        tmem_wait_st();
        tc_fence_before();
      }
      if (need) {
#pragma unroll
        for (int e = 0; e < 128; ++e) v[e] -= mt;
        ref = r0 + mt;
      }
      l *= f;
    }
    // the exponentials (the pairs kEmuMask names on the FMA pipe), then the wait for the P buffer,
    // then the stores
    uint32_t pk[64];
    float sum = 0.f;
#pragma unroll
    for (int e = 0; e < 64; ++e) {
      const bool emu = ((kEmuMask >> (e & 7)) & 1) != 0;
      const float p0 = emu ? ex2_poly<3>(v[2 * e]) : ex2_approx(v[2 * e]);
      const float p1 = emu ? ex2_poly<3>(v[2 * e + 1]) : ex2_approx(v[2 * e + 1]);
      sum += p0 + p1;
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
      pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
    }
    l += sum;
    if (!pv_done && !mbar_wait(&s.p_empty[x], (j - 1) & 1, &s.abort, wait_ns)) {
      fail(s, p, 0x923);
      return;
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      char* dst = reinterpret_cast<char*>(&s.p[x][hh][0]) + row * 128;
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        const int e = 32 * hh + 4 * c8;
        *reinterpret_cast<uint4*>(dst + ((c8 ^ (row & 7)) << 4)) = make_uint4(pk[e], pk[e + 1], pk[e + 2], pk[e + 3]);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && !(p.skip_arrive && x == 0 && j == 0)) mbar_arrive(&s.p_full[x]);
  }
  // epilogue: O / l -> bf16 -> global
  if (!mbar_wait(&s.o_full[x], 0, &s.abort, wait_ns)) {
    fail(s, p, 0x924);
    return;
  }
  tc_fence_after();
  const float inv = (row_ok && l > 0.f) ? 1.f / l : 0.f;
  __nv_bfloat16* orow = p.O + ((size_t)h * p.total_q + pr.q0 + qi) * 128;
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    uint32_t xs[32];
    tmem_ld32(tbase + lane_addr + o_col + 32 * c, xs);
    tmem_wait_ld();
    if (row_ok && checked(p.ws, h < p.H && pr.q0 + qi < p.total_q, 0xC41)) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t q[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(xs[8 * g + 2 * e]) * inv,
                                                          __uint_as_float(xs[8 * g + 2 * e + 1]) * inv);
          q[e] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        *reinterpret_cast<uint4*>(orow + 32 * c + 8 * g) = make_uint4(q[0], q[1], q[2], q[3]);
      }
    }
  }
  tc_fence_before();
}

__global__ void __launch_bounds__(kThreads, 1)
    k_dense_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
               const __grid_constant__ CUtensorMap tv, Params p) {
  Pair pr;
  if (!find_pair(p, (int)blockIdx.x, pr)) return;  // past the last pair: the whole CTA leaves
  const int h = (int)blockIdx.y;
  extern __shared__ unsigned char smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&s.q_full, 1);
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&s.slot_full[i], 1);
      mbar_init(&s.slot_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.s_empty[i], 4);
      mbar_init(&s.p_full[i], 4);
      mbar_init(&s.p_empty[i], 1);
      mbar_init(&s.o_full[i], 1);
    }
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
  if (warp < kSoftmaxWarp0) {
    regs_dec<kRegsControl>();
    if (warp == kProducerWarp)
      producer(s, p, pr, h, &tq, &tk, &tv);
    else if (warp == kMmaWarp)
      mma_issuer(s, p, pr);
  } else {
    regs_inc<kRegsSoftmax>();
    const int x = (warp - kSoftmaxWarp0) >> 2;
    if (pr.nk[x] > 0) softmax_group(s, p, pr, h, x);  // a one-tile pair leaves warpgroup B idle
  }
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
  // the register split assumes the launch allocation it was sized for; anything else could leave
  // an increase waiting for registers that do not exist
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, k_dense_tc);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidConfiguration;
  const size_t smem = sizeof(Smem) + 1024;
  e = cudaFuncSetAttribute(k_dense_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // pairs of all sequences: sum of ceil(tiles / 2) <= total_q / 256 + n_seq; CTAs past the last leave
  dim3 grid((unsigned)(a.total_q / 256 + a.n_seq), (unsigned)a.H);
  ProfScope ps(kKDenseTc, a.stream);
  k_dense_tc<<<grid, kThreads, smem, a.stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace mr
