// Fused translated retrieval on sm_100a (bf16 maps, d_v = 128): MapFlow section 5.4.
//
//   O_r[i] = sum_J X_r[I, J] V_r[J],   X_r[I, J] = sum_s W[r, s] A_s[I, J]  (kept tiles only)
//
// One CTA per SM walks a static, longest-first list of units.  A unit is 128 query rows (one
// query block of 128, or two consecutive blocks of 64) x G receiver heads x R requests, with
// G * R = 4 fp32 accumulators of 128 x 128 in Tensor Memory (all 512 columns).  Key blocks are
// consumed in sub-steps of 64 keys:
//   * producer warp: for every sender head that kept the key block (bitmask union), bulk-copies
//     that tile's 64-column panel (a 128-byte-swizzled K-major operand as stored) into a ring of
//     shared-memory slots, and loads the receivers' V rows with TMA (128-byte swizzle);
//   * 8 mixer warps: the head mixing as a weighted accumulation in registers (each thread owns
//     one row and 32 columns for G heads), then write X_r as a bf16 MMA operand to shared memory;
//     the translated map exists only there, never in global memory;
//   * MMA warp: tcgen05.mma X_r (128 x 64, K-major) x V (64 x 128, MN-major) into the fp32
//     accumulators;
//   * epilogue (mixer warps): Tensor Memory -> registers -> bf16 -> global O.
// Every wait is bounded; a wait that runs out records MR_ERR_TIMEOUT and the CTA drains its
// in-flight copies and MMAs, frees Tensor Memory and returns.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "profile.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace mr {
namespace {

using namespace sm100;

constexpr int kMixWarps = 8;
constexpr int kProducerWarp0 = 8;  // producer warps 8, 9, 10 (each owns ring slots p and p + 3)
constexpr int kProducers = 3;
constexpr int kMmaWarp = 11;
constexpr int kThreads = 384;
constexpr int kSlots = 6;
constexpr int kSlotBytes = 16384;
constexpr int kAcc = 4;
constexpr uint64_t kTimeoutNs = 2000000000ull;

struct Params {
  const uint32_t* kept_bits;
  const int32_t* row_ptr;
  const __nv_bfloat16* vals;
  int64_t capacity;
  const float* W;
  __nv_bfloat16* O;
  const int64_t* v_req_off;
  int64_t v_req_stride, v_head_stride;
  int H_s, H_r, L, B, nqb, nkw, n_req;
  int R, n_hg, n_rg, n_rb, n_units;
  WsHeader* ws;
};

// What a ring slot holds, written by the producer before the slot's full barrier is armed.
struct SlotMeta {
  float w[kAcc];   // W[r][s] of the unit's receiver heads for the slot's sender head s
  uint32_t flags;  // kHalf0 | kHalf1 | kLastSub | kLastUnit | kEmptyUnit
};
constexpr uint32_t kHalf0 = 1u, kHalf1 = 2u, kLastSub = 4u, kLastUnit = 8u, kEmptyUnit = 16u;

struct Smem {
  __nv_bfloat16 slot[kSlots][kSlotBytes / 2];
  __nv_bfloat16 x[kAcc][128 * 64];
  __nv_bfloat16 v[kAcc][64 * 128];
  SlotMeta meta[kSlots];
  uint64_t slot_full[kSlots];
  uint64_t slot_empty[kSlots];
  uint64_t x_full, x_empty, v_full, v_empty, o_full, o_empty, mma_done;
  uint32_t tmem_base;
  int abort;
};

struct Unit {
  int rb, hg, rg, I0, I1, Jmax;
};

__device__ __forceinline__ Unit decode(const Params& p, int k) {
  const int per = p.n_hg * p.n_rg;
  Unit u;
  u.rb = p.n_rb - 1 - k / per;
  const int rest = k % per;
  u.hg = rest % p.n_hg;
  u.rg = rest / p.n_hg;
  if (p.B == 128) {
    u.I0 = u.rb;
    u.I1 = -1;
    u.Jmax = u.rb;
  } else {
    u.I0 = 2 * u.rb;
    u.I1 = (2 * u.rb + 1 < p.nqb) ? 2 * u.rb + 1 : -1;
    u.Jmax = u.I1 >= 0 ? u.I1 : u.I0;
  }
  return u;
}

// Warp-collective: bit s set iff sender head s kept key block J in query block I.
__device__ __forceinline__ uint64_t head_mask(const Params& p, int I, int J) {
  const int lane = threadIdx.x & 31;
  bool b0 = false, b1 = false;
  if (I >= 0 && J <= I) {
    const int wj = J >> 5, bj = J & 31;
    if (lane < p.H_s) b0 = (__ldg(p.kept_bits + (size_t)(lane * p.nqb + I) * p.nkw + wj) >> bj) & 1u;
    if (lane + 32 < p.H_s) b1 = (__ldg(p.kept_bits + (size_t)((lane + 32) * p.nqb + I) * p.nkw + wj) >> bj) & 1u;
  }
  const uint32_t lo = __ballot_sync(0xffffffffu, b0);
  const uint32_t hi = __ballot_sync(0xffffffffu, b1);
  return ((uint64_t)hi << 32) | lo;
}

__device__ __forceinline__ bool acc_valid(const Params& p, const Unit& u, int G, int a) {
  const int g = a / p.R, q = a % p.R;
  return u.hg * G + g < p.H_r && u.rg * p.R + q < p.n_req;
}

__device__ __forceinline__ void fail(Smem& s, const Params& p, uint32_t detail) {
  set_status(p.ws, MR_ERR_TIMEOUT, detail);
  s.abort = 1;
}

// ------------------------------------------------------------------------------------------------
// Per-lane view of one (sender head, query block) map row while J advances within a unit: the
// current 32-bit word of kept bits, the number of kept blocks below J, and the row's first tile.
struct RowCursor {
  const uint32_t* bits;
  uint32_t word;
  int count;
  int64_t first;
  bool live;
  __device__ __forceinline__ void start(const Params& p, int s, int I) {
    live = s < p.H_s && I >= 0;
    count = 0;
    if (live) {
      const int row = s * p.nqb + I;
      bits = p.kept_bits + (size_t)row * p.nkw;
      word = __ldg(bits);
      first = __ldg(p.row_ptr + row);
    } else {
      bits = nullptr;
      word = 0u;
      first = 0;
    }
  }
  // kept flag of block J (J visited in increasing order, J <= I of the row)
  __device__ __forceinline__ bool at(int J) {
    if (!live) return false;
    if ((J & 31) == 0 && J > 0) word = __ldg(bits + (J >> 5));
    return (word >> (J & 31)) & 1u;
  }
};

// Producer warp `pw` (0..2).  Bulk copies are issued by several warps because one issuing warp
// is limited to a few million copies per second; each warp fills only the ring slots it owns
// (slot % 3 == pw), so a slot's fills are always issued by one warp, in order, each after the
// release of the previous one.  All producer warps walk the same unit / key-block sequence.
template <int G>
__device__ void producer(Smem& s, const Params& p, const CUtensorMap* tmap_v, int pw) {
  const int lane = threadIdx.x & 31;
  uint32_t f = 0;   // slot fills in the sequence so far (all warps)
  uint32_t nv = 0;  // V fills issued (warp 0 only; one per executed sub-step)
  uint32_t hi = 0;  // one past the last fill this warp issued
  const int nparts = p.B / 64;
  bool ok = true;

  auto issue_v = [&](const Unit& u, int j0) {
    uint32_t bytes = 0;
    for (int a = 0; a < G * p.R; ++a)
      if (acc_valid(p, u, G, a)) bytes += 64 * 128 * 2;
    mbar_arrive_expect_tx(&s.v_full, bytes);
    for (int a = 0; a < G * p.R; ++a) {
      if (!acc_valid(p, u, G, a)) continue;
      const int r = u.hg * G + a / p.R, q = u.rg * p.R + a % p.R;
      const int64_t off = (p.v_req_off ? p.v_req_off[q] : (int64_t)q * p.v_req_stride) + (int64_t)r * p.v_head_stride;
      const int row = (int)(off / 128) + j0;
      tma_load_2d(&s.v[a][0], tmap_v, &s.v_full, 0, row);
      tma_load_2d(&s.v[a][64 * 64], tmap_v, &s.v_full, 64, row);
    }
    ++nv;
  };
  auto owns = [&](uint32_t F) { return (int)((F % kSlots) % kProducers) == pw; };
  // lane 0 waits until the slot of fill F is free (its previous fill, issued by this warp, released)
  auto claim = [&](uint32_t F) -> bool {
    bool good = true;
    if (lane == 0 && F >= (uint32_t)kSlots &&
        !mbar_wait(&s.slot_empty[F % kSlots], ((F / kSlots) - 1) & 1, &s.abort, kTimeoutNs)) {
      fail(s, p, 0x102);
      good = false;
    }
    return __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
  };

  for (int k = blockIdx.x; k < p.n_units && ok; k += gridDim.x) {
    const Unit u = decode(p, k);
    // lane l tracks sender heads l and l + 32, for the unit's one or two query blocks
    RowCursor cur[2][2];
    float wv[2][kAcc];
#pragma unroll
    for (int hs = 0; hs < 2; ++hs) {
      const int sh = lane + 32 * hs;
      cur[0][hs].start(p, sh, u.I0);
      cur[1][hs].start(p, sh, p.B == 64 ? u.I1 : -1);
#pragma unroll
      for (int g = 0; g < kAcc; ++g) {
        const int r = u.hg * G + g;
        wv[hs][g] = (g < G && sh < p.H_s && r < p.H_r) ? __ldg(p.W + (size_t)r * p.H_s + sh) : 0.f;
      }
    }
    bool any_unit = false;
    for (int J = 0; J <= u.Jmax && ok; ++J) {
      bool b[2][2];
#pragma unroll
      for (int pt = 0; pt < 2; ++pt)
#pragma unroll
        for (int hs = 0; hs < 2; ++hs) {
          const int I = pt == 0 ? u.I0 : u.I1;
          b[pt][hs] = (pt == 0 || p.B == 64) && I >= 0 && J <= I ? cur[pt][hs].at(J) : false;
        }
      const uint64_t m0 = ((uint64_t)__ballot_sync(0xffffffffu, b[0][1]) << 32) | __ballot_sync(0xffffffffu, b[0][0]);
      const uint64_t m1 = p.B == 64
                              ? (((uint64_t)__ballot_sync(0xffffffffu, b[1][1]) << 32) | __ballot_sync(0xffffffffu, b[1][0]))
                              : m0;
      const uint64_t uni = m0 | m1;
      if (uni != 0) {
        const int nsl = __popcll((long long)uni);
        for (int h = 0; h < nparts && ok; ++h) {
          const int j0 = J * p.B + 64 * h;
          uint64_t rem = uni;
          for (int rank = 0; rank < nsl && ok; ++rank) {
            const int sh = __ffsll((long long)rem) - 1;
            rem &= rem - 1;
            const uint32_t F = f + (uint32_t)rank;
            if (!owns(F)) continue;  // warp-uniform
            if (!claim(F)) {
              ok = false;
              break;
            }
            const int src_lane = sh & 31, hs = sh >> 5;
            int64_t t[2];
            bool use[2];
#pragma unroll
            for (int pt = 0; pt < 2; ++pt) {
              const int64_t t0 = __shfl_sync(0xffffffffu, cur[pt][0].first + cur[pt][0].count, src_lane);
              const int64_t t1 = __shfl_sync(0xffffffffu, cur[pt][1].first + cur[pt][1].count, src_lane);
              t[pt] = hs ? t1 : t0;
              use[pt] = ((pt == 0 ? m0 : m1) >> sh) & 1ull;
            }
            float w[kAcc];
#pragma unroll
            for (int g = 0; g < kAcc; ++g) {
              const float w0 = __shfl_sync(0xffffffffu, wv[0][g], src_lane);
              const float w1 = __shfl_sync(0xffffffffu, wv[1][g], src_lane);
              w[g] = hs ? w1 : w0;
            }
            if (lane == 0) {
              const int slot = (int)(F % kSlots);
              char* dst = reinterpret_cast<char*>(&s.slot[slot][0]);
              uint32_t bytes = 0, flags = 0;
              const uint32_t len = p.B == 128 ? 16384u : 8192u;
              const char* src[2] = {nullptr, nullptr};
              for (int pt = 0; pt < (p.B == 64 ? 2 : 1); ++pt) {
                if (!use[pt]) continue;
                flags |= pt == 0 ? kHalf0 : kHalf1;
                if (t[pt] >= p.capacity) {
                  // the map overflowed: this tile was never stored; contribute zeros
                  uint4* z = reinterpret_cast<uint4*>(dst + pt * 8192);
                  for (uint32_t e = 0; e < len / 16; ++e) z[e] = make_uint4(0, 0, 0, 0);
                  set_status(p.ws, MR_ERR_CAPACITY, 3u);
                } else {
                  src[pt] = reinterpret_cast<const char*>(p.vals + t[pt] * (int64_t)p.B * p.B) + (p.B == 128 ? 16384 * h : 0);
                  bytes += len;
                }
              }
              if (p.B == 128) flags |= kHalf1;  // one 128-row panel serves every row
              if (rank == nsl - 1) flags |= kLastSub;
#pragma unroll
              for (int g = 0; g < kAcc; ++g) s.meta[slot].w[g] = w[g];
              s.meta[slot].flags = flags;
              mbar_arrive_expect_tx(&s.slot_full[slot], bytes);
              for (int pt = 0; pt < 2; ++pt)
                if (src[pt]) bulk_g2s(dst + pt * 8192, src[pt], len, &s.slot_full[slot]);
            }
            hi = F + 1;
            __syncwarp();
          }
          if (!ok) break;
          f += (uint32_t)nsl;
          // V of this sub-step (warp 0), once the previous sub-step's MMAs released the V buffer
          if (pw == 0 && lane == 0) {
            if (nv > 0 && !mbar_wait(&s.v_empty, (nv - 1) & 1, &s.abort, kTimeoutNs)) {
              fail(s, p, 0x101);
              ok = false;
            } else {
              issue_v(u, j0);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          nv = __shfl_sync(0xffffffffu, nv, 0);
          any_unit = true;
        }
      }
      // advance the kept counts past block J
#pragma unroll
      for (int pt = 0; pt < 2; ++pt)
#pragma unroll
        for (int hs = 0; hs < 2; ++hs) cur[pt][hs].count += b[pt][hs] ? 1 : 0;
    }
    if (!ok) break;
    // mark the end of the unit with a data-less slot (the unit's only slot if it kept nothing)
    if (owns(f)) {
      if (!claim(f)) {
        ok = false;
        break;
      }
      if (lane == 0) {
        s.meta[f % kSlots].flags = any_unit ? kLastUnit : (kLastUnit | kEmptyUnit);
        mbar_arrive(&s.slot_full[f % kSlots]);
      }
      hi = f + 1;
      __syncwarp();
    }
    ++f;
  }
  // drain: every copy this warp issued must land before the CTA can release its shared memory
  if (lane == 0) {
    const int never = 0;  // drain even after an abort: wait on the copies themselves (bounded)
    for (uint32_t g = (hi > (uint32_t)kSlots ? hi - kSlots : 0); g < hi; ++g)
      if (owns(g)) mbar_wait(&s.slot_full[g % kSlots], (g / kSlots) & 1, &never, kTimeoutNs);
    if (nv > 0) mbar_wait(&s.v_full, (nv - 1) & 1, &never, kTimeoutNs);
  }
  __syncwarp();
}

template <int G>
__device__ void mma_issuer(Smem& s, const Params& p) {
  const int lane = threadIdx.x & 31;
  const uint32_t idesc = idesc_bf16_f32(128, 128, false, true);
  const uint32_t tbase = s.tmem_base;
  uint32_t nsub = 0;
  int nunit = 0;
  bool ok = true;
  const int nparts = p.B / 64;
  for (int k = blockIdx.x; k < p.n_units && ok; k += gridDim.x, ++nunit) {
    const Unit u = decode(p, k);
    if (lane == 0 && nunit > 0 && !mbar_wait(&s.o_empty, (nunit - 1) & 1, &s.abort, kTimeoutNs)) {
      fail(s, p, 0x201);
      ok = false;
    }
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (!ok) break;
    bool first = true;
    for (int J = 0; J <= u.Jmax && ok; ++J) {
      const uint64_t m0 = head_mask(p, u.I0, J);
      const uint64_t m1 = (p.B == 64) ? head_mask(p, u.I1, J) : m0;
      if ((m0 | m1) == 0) continue;
      for (int h = 0; h < nparts && ok; ++h) {
        if (lane == 0) {
          if (!mbar_wait(&s.x_full, nsub & 1, &s.abort, kTimeoutNs) ||
              !mbar_wait(&s.v_full, nsub & 1, &s.abort, kTimeoutNs)) {
            fail(s, p, 0x202);
            ok = false;
          } else {
            tc_fence_after();
            for (int a = 0; a < G * p.R; ++a) {
              if (!acc_valid(p, u, G, a)) continue;
              const int g = a / p.R;
              const uint32_t xa = smem_u32(&s.x[g][0]);
              const uint32_t va = smem_u32(&s.v[a][0]);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t da = sdesc_sw128(xa + 32 * kk, 16, 1024);
                const uint64_t dv = sdesc_sw128(va + 2048 * kk, 8192, 1024);
                mma_bf16_ss(tbase + 128 * a, da, dv, idesc, (first && kk == 0) ? 0u : 1u);
              }
            }
            mma_commit(&s.x_empty);
            mma_commit(&s.v_empty);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        first = false;
        ++nsub;
      }
    }
    if (ok && lane == 0) {
      if (first)
        mbar_arrive(&s.o_full);  // nothing accumulated: the epilogue writes zeros
      else
        mma_commit(&s.o_full);
    }
    __syncwarp();
  }
  // drain: all MMAs issued by this thread complete before Tensor Memory is released
  if (lane == 0) {
    mma_commit(&s.mma_done);
    const int never = 0;
    mbar_wait(&s.mma_done, 0, &never, kTimeoutNs);
  }
  __syncwarp();
}

// ------------------------------------------------------------------------------------------------
// What a mixer thread takes from one ring slot: the slot's flags and weights and its own 32
// columns of its own row (4 x 16 bytes).
struct SlotData {
  uint32_t flags;
  float w[kAcc];
  uint4 d[4];
};

template <int G>
__device__ void mixers(Smem& s, const Params& p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = 32 * (warp & 3) + lane;  // 0..127: this thread's query row within the unit
  const int chalf = warp >> 2;             // which 32 of the sub-step's 64 columns
  const int half = row >> 6;               // for 64-key blocks: which of the two query blocks
  const uint32_t use_mask = (p.B == 128) ? kHalf1 : (half ? kHalf1 : kHalf0);
  const uint32_t row_off = (p.B == 64) ? (uint32_t)(half * 8192 + (row & 63) * 128) : (uint32_t)(row * 128);
  const int sw = row & 7;
  const uint32_t tbase = s.tmem_base;
  uint32_t fetched = 0, nsub = 0;
  int nunit = 0;
  bool ok = true;

  // Wait for the next fill, copy what this thread needs into registers, and hand the slot back
  // to the producer at once (the arrive orders the reads before any refill).
  auto fetch = [&](SlotData& o) -> bool {
    const int slot = (int)(fetched % kSlots);
    if (!mbar_wait(&s.slot_full[slot], (fetched / kSlots) & 1, &s.abort, kTimeoutNs)) return false;
    o.flags = s.meta[slot].flags;
#pragma unroll
    for (int g = 0; g < G; ++g) o.w[g] = s.meta[slot].w[g];
    if (!(o.flags & kLastUnit) && (o.flags & use_mask)) {
      const char* base = reinterpret_cast<const char*>(&s.slot[slot][0]) + row_off;
#pragma unroll
      for (int c = 0; c < 4; ++c) o.d[c] = *reinterpret_cast<const uint4*>(base + (((4 * chalf + c) ^ sw) << 4));
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.slot_empty[slot]);
    ++fetched;
    return true;
  };

  unsigned long long acc[G][16];  // pairs of fp32 accumulators: columns (2e, 2e + 1)
  SlotData cur;
  for (int k = blockIdx.x; k < p.n_units && ok; k += gridDim.x, ++nunit) {
    const Unit u = decode(p, k);
    bool any = false, unit_done = false;
    while (!unit_done && ok) {
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[g][e] = 0ull;
      bool sub_done = false;
      while (!sub_done) {
        if (!fetch(cur)) {
          fail(s, p, 0x301);
          ok = false;
          break;
        }
        const bool marker = (cur.flags & kLastUnit) != 0;
        if (marker) {
          unit_done = true;
          break;
        }
        if (cur.flags & use_mask) {
          unsigned long long w2[G];
#pragma unroll
          for (int g = 0; g < G; ++g) w2[g] = pack2(cur.w[g], cur.w[g]);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t wd[4] = {cur.d[c].x, cur.d[c].y, cur.d[c].z, cur.d[c].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const unsigned long long v2 =
                  pack2(__uint_as_float(wd[e] << 16), __uint_as_float(wd[e] & 0xffff0000u));
#pragma unroll
              for (int g = 0; g < G; ++g) acc[g][4 * c + e] = ffma2(w2[g], v2, acc[g][4 * c + e]);
            }
          }
        }
        sub_done = (cur.flags & kLastSub) != 0;
      }
      if (!ok || unit_done) break;
      any = true;
      // hand X to the tensor core once the previous sub-step's MMAs have read it
      if (nsub > 0 && !mbar_wait(&s.x_empty, (nsub - 1) & 1, &s.abort, kTimeoutNs)) {
        fail(s, p, 0x302);
        ok = false;
        break;
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        char* xb = reinterpret_cast<char*>(&s.x[g][0]) + row * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float lo, hi;
            unpack2(acc[g][4 * c + e], lo, hi);
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(lo, hi);
            pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          *reinterpret_cast<uint4*>(xb + (((4 * chalf + c) ^ sw) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.x_full);
      ++nsub;
    }
    if (!ok) break;
    // ---- epilogue: accumulators -> bf16 -> O ----
    if (!mbar_wait(&s.o_full, nunit & 1, &s.abort, kTimeoutNs)) {
      fail(s, p, 0x303);
      ok = false;
      break;
    }
    tc_fence_after();
    const int i = u.rb * 128 + row;
    for (int a = chalf; a < G * p.R; a += 2) {
      const bool valid = acc_valid(p, u, G, a);
      const int r = u.hg * G + a / p.R, q = u.rg * p.R + a % p.R;
      __nv_bfloat16* orow = p.O + (((size_t)q * p.H_r + r) * p.L + i) * 128;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        tmem_ld32(tbase + ((uint32_t)(32 * (warp & 3)) << 16) + 128 * a + 32 * cc, v);
        tmem_wait_ld();
        if (valid && i < p.L) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = any ? __uint_as_float(v[8 * c + 2 * e]) : 0.f;
              const float x1 = any ? __uint_as_float(v[8 * c + 2 * e + 1]) : 0.f;
              const __nv_bfloat162 b2 = __floats2bfloat162_rn(x0, x1);
              pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            *reinterpret_cast<uint4*>(orow + 32 * cc + 8 * c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.o_empty);
  }
}

template <int G>
__global__ void __launch_bounds__(kThreads, 1) k_retrieve_tc(const __grid_constant__ CUtensorMap tmap_v, Params p) {
  extern __shared__ unsigned char smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&s.slot_full[i], 1);
      mbar_init(&s.slot_empty[i], kMixWarps);
    }
    mbar_init(&s.x_full, kMixWarps);
    mbar_init(&s.x_empty, 1);
    mbar_init(&s.v_full, 1);
    mbar_init(&s.v_empty, 1);
    mbar_init(&s.o_full, 1);
    mbar_init(&s.o_empty, kMixWarps);
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
  if (warp < kMixWarps)
    mixers<G>(s, p);
  else if (warp < kProducerWarp0 + kProducers)
    producer<G>(s, p, &tmap_v, warp - kProducerWarp0);
  else
    mma_issuer<G>(s, p);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(s.tmem_base, 512);
}

template <int G>
cudaError_t launch_g(const RetrieveArgs& a, const Params& p, const CUtensorMap& tm, int grid, cudaStream_t st) {
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(k_retrieve_tc<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps(kKRetrieveTc, st);
  k_retrieve_tc<G><<<grid, kThreads, smem, st>>>(tm, p);
  return cudaGetLastError();
}

}  // namespace

bool tc_retrieve_supported(const RetrieveArgs& a) {
  return a.dt == MR_BF16 && a.d_v == 128 && (a.map.block == 64 || a.map.block == 128) && a.map.H_s <= 64 &&
         a.v_head_stride % 128 == 0 && (a.v_req_off != nullptr || a.v_req_stride % 128 == 0);
}

cudaError_t tc_retrieve(const RetrieveArgs& a) {
  Params p;
  p.kept_bits = a.map.kept_bits;
  p.row_ptr = a.map.row_ptr;
  p.vals = (const __nv_bfloat16*)a.map.vals;
  p.capacity = a.map.capacity_tiles;
  p.W = a.W;
  p.O = (__nv_bfloat16*)a.O;
  p.v_req_off = a.v_req_off;
  p.v_req_stride = a.v_req_stride;
  p.v_head_stride = a.v_head_stride;
  p.H_s = a.map.H_s;
  p.H_r = a.H_r;
  p.L = a.map.L;
  p.B = a.map.block;
  p.nqb = a.map.L / a.map.block;
  p.nkw = (p.nqb + 31) / 32;
  p.n_req = a.n_req;
  int G = 4;
  if (a.n_req >= 4)
    G = 1;
  else if (a.n_req >= 2)
    G = 2;
  p.R = kAcc / G;
  p.n_hg = (a.H_r + G - 1) / G;
  p.n_rg = (a.n_req + p.R - 1) / p.R;
  p.n_rb = (a.map.L + 127) / 128;
  p.n_units = p.n_rb * p.n_hg * p.n_rg;
  p.ws = a.ws;
  // V viewed as rows of 128 bf16; rows are addressed from the request offset and head stride.
  // With strided requests the exact extent is known (rows past it read as zeros); with a device
  // offset table it is not, and the view spans the 32-bit row range.
  CUtensorMap tm;
  uint64_t rows = ((uint64_t)1 << 31) - 1;
  if (a.v_req_off == nullptr)
    rows = (uint64_t)(((int64_t)(a.n_req - 1) * a.v_req_stride + (int64_t)(a.H_r - 1) * a.v_head_stride) / 128) +
           (uint64_t)a.map.L;
  if (!make_tmap_bf16_2d(&tm, a.V, 128, rows, 256, 64, 64)) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = p.n_units < sms ? p.n_units : sms;
  if (G == 4) return launch_g<4>(a, p, tm, grid, a.stream);
  if (G == 2) return launch_g<2>(a, p, tm, grid, a.stream);
  return launch_g<1>(a, p, tm, grid, a.stream);
}

}  // namespace mr
