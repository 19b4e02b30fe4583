// Fused translated retrieval on sm_100a (bf16 maps, d_v = 128): MapFlow section 5.4.
//
//   O_r[i] = sum_J X_r[I, J] V_r[J],   X_r[I, J] = sum_s W[r, s] A_s[I, J]  (kept tiles only)
//
// One CTA per SM walks a static, longest-first list of units.  A unit is 128 query rows (one
// query block of 128, or two consecutive blocks of 64) x G receiver heads x R requests, with
// G * R = 4 fp32 accumulators of 128 x 128 in Tensor Memory (all 512 columns).  Key blocks are
// consumed in sub-steps of 64 keys:
//   * planner warp: for every sender head that kept the key block (bitmask union) writes one
//     entry (tile index, the unit's mixing weights W[r, s]) into a page of a shared-memory ring,
//     one page per sub-step, and pulls the sub-step's map panels into L2 ahead of use;
//   * mixer warps copy the listed panels from L2 into private shared-memory rings (cp.async,
//     per-thread completion: no per-panel barrier), mix the sender heads, and write X_r as a bf16
//     MMA operand to shared memory; the translated map exists only there, never in global memory.
//     bf16 maps of 128-key blocks with at most 32 sender heads and 4 receiver heads per CTA: 8
//     warps mix on the tensor core, one unit row x 16 sender heads per mma.sync step with fp32
//     register accumulators (Tensor Memory holds the Ã·V accumulators).  Otherwise: 16 warps,
//     each thread mixing its own 2 x 16 bytes of every listed panel in fp32 (pairs of columns per
//     FFMA2) or, for fp8 maps, in pre-scaled half precision;
//   * MMA warp: loads the receivers' V rows for the next sub-step with TMA (128-byte swizzle)
//     once the current MMAs have read the buffer, and issues tcgen05.mma X_r (128 x 64, K-major)
//     x V (64 x 128, MN-major) into the fp32 accumulators;
//   * epilogue (mixer warps): Tensor Memory -> registers -> bf16 -> global O.
// Every wait is bounded; a wait that runs out records MR_ERR_TIMEOUT and the CTA drains its
// in-flight copies and MMAs, frees Tensor Memory and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"
#include "profile.h"
#include "sm100.cuh"
#include "tma_host.h"

namespace mr {
namespace {

using namespace sm100;

// CUDA-core mixing: 16 mixer warps + planner + MMA warp.  Five warps then share one SM
// sub-partition, which caps a thread at 96 registers: enough for 4 x 16 fp32 accumulators (2
// pieces per thread) with the paired FMA as a compiler builtin.  Measured against 8 mixer warps
// with 4 pieces each (168 registers): 4 mixer warps per sub-partition hide more latency, 5% faster
// at 32K tokens.
constexpr int kMixWarps = 16;  // CUDA-core mixing path (the tensor-core one runs 8, see Roles)
constexpr int kMixThreads = kMixWarps * 32;
constexpr int kRowsW = 128 / kMixWarps;                  // unit rows per mixer warp
constexpr int kPieces = 128 * 8 / kMixThreads;           // 16-byte pieces per thread per panel
// entry pairs in flight per mixer thread (its shared-memory ring): an fp8 piece is half the bytes,
// so the same ring holds twice the pairs
template <bool F8>
__host__ __device__ constexpr int queue_of() { return F8 ? 4 : 2; }
constexpr int kMaxEntries = 64; // sender heads
constexpr uint32_t kMmSlots = 6;  // tensor-core mixing: 2 KB ring slots per mixer warp
constexpr int kPaceSlack = 4;   // pages a CTA may run ahead of the slowest CTA of its group
constexpr uint64_t kPaceNs = 100000ull;  // longest hold per page
constexpr int kAcc = 4;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr uint32_t kNone = 0xffffffffu;

struct Params {
  const uint32_t* kept_bits;
  const int32_t* row_ptr;
  const __nv_bfloat16* vals;
  const uint8_t* vals8;      // fp8 (e4m3) maps
  const float* tile_scale;   // fp8 maps: one scale per 32-row x 64-key piece
  int64_t capacity;
  const float* W;
  __nv_bfloat16* O;
  const int64_t* v_req_off;
  int64_t v_req_stride, v_head_stride;
  int64_t v_rows;  // rows of 128 values in the V allocation (the tensor map's extent)
  int v_group;     // receiver heads per value head
  int H_v;         // value heads
  const int32_t* v_pages;  // paged values: [n_req][pages_per_req] page numbers, or nullptr
  int page_rows, pages_per_req;
  int H_s, H_r, L, B, nqb, nkw, n_req;
  int R, n_hg, n_rg, n_rb, n_units;
  int rb_hi;       // 128-row blocks rb_hi - n_rb .. rb_hi - 1 hold the output query blocks
  int qb0, qb1;    // output query blocks qb0 <= I < qb1
  int per;      // units per row block: head groups x request groups
  int groups;   // > 0: grouped schedule with this many groups of `per` CTAs (one wave)
  uint32_t* progress;  // [gridDim.x] pages consumed by each CTA's mixers (workspace, zeroed)
  WsHeader* ws;
};

// One listed panel: the tile of each of the unit's two query blocks (kNone: not kept, or never
// stored because the map overflowed) and the unit's mixing weights for the panel's sender head.
template <bool SC>
struct EntryT {
  uint32_t t[2];
  uint32_t sc[2];  // fp8 maps: the scale of each 32-row group q of the unit in this panel, as bf16
                   // (group q in half q % 2 of word q / 2); unused for bf16 maps
  float w[kAcc];
};
template <>
struct EntryT<false> {  // the tensor-core mixing's entries (bf16 maps): no scales
  uint32_t t[2];
  float w[kAcc];
};
using Entry = EntryT<true>;
// One sub-step (n >= 1 entries, panel h of the key block) or a marker (n == 0).
template <int E, bool SC>
struct PageT {
  uint32_t n, h, flags, pad;
  EntryT<SC> e[E];
};
constexpr uint32_t kUnitEnd = 1u, kEmptyUnit = 2u, kEnd = 4u;

// fp8 maps: one 16-key piece of one row per thread and panel (a 64-key panel row is 64 bytes), and
// the piece's scale next to it; values are mixed in half precision pre-scaled by 2^14 (so they stay
// in its normal range; a mixed value is at most 2^14), undone exactly in the epilogue.
constexpr int kPieces8 = 1;
constexpr float kF8Pre = 16384.f;
constexpr float kF8Decode = 256.f;  // the integer decode yields value * 2^-8

// Shared memory of the CUDA-core mixing (MM = false); the tensor-core mixing has its own layout below.
template <bool F8, bool MM>
struct SmemT {
  // > 2 * queue_of<true>() + 2 pages, so the fetch cursor never laps the compute cursor
  static constexpr int kPages = 12;
  using Page = PageT<kMaxEntries, true>;
  // X of each accumulator (bf16 MMA operand, 128 rows x 64 keys, 128-byte swizzle).  Each buffer
  // starts 128 bytes further into the swizzle pattern than the one before, so the same row and
  // chunk of the receivers' buffers fall in different banks.  The tensor core applies the swizzle
  // to absolute shared-memory addresses (as TMA does): row r of buffer a has phase (r + a) % 8 and
  // the descriptor is the plain one (measured: a base offset of a in the descriptor reads wrong data).
  __nv_bfloat16 x[kAcc][128 * 64 + 64];
  char x_align[1024 - kAcc * 128 % 1024];  // V on a 1024-byte boundary
  __nv_bfloat16 v[kAcc][64 * 128];
  uint4 ring[queue_of<F8>() * 2 * (F8 ? kPieces8 : kPieces) * kMixThreads];  // [pair slot][entry][piece][mixer thread]
  Page page[kPages];
  uint64_t plan_full[kPages], plan_empty[kPages];
  uint64_t x_full, x_empty, v_full, v_empty, o_full, o_empty, mma_done;
  uint32_t tmem_base;
  int abort;
};
// The tensor-core mixing (bf16 maps, at most 32 sender heads) fills the opt-in limit: V first (on
// the 1024-byte boundary its swizzle needs), then the staggered X buffers, whose 128-byte gaps take
// the zero rows of the matrix stores, a ring of kMmSlots 2 KB slots per mixer warp, and three pages
// of 32 entries.  Three pages suffice: the fetch cursor is at most one page (kMmSlots steps < 16)
// and one unit-end marker ahead of the compute cursor, and at 128-key blocks no unit is empty
// (every query row sees its own key, a logit no bias masks, so with p > 0 every head keeps a
// block of every query block), so markers never follow one another (the final end marker follows
// a unit-end marker, which is the one marker and page the cursor may pass).  The launch adds no alignment slack; the kernel checks that
// its dynamic shared memory starts on a 1024-byte boundary.
template <bool F8>
struct SmemT<F8, true> {
  static constexpr int kPages = 3;
  using Page = PageT<32, false>;
  __nv_bfloat16 v[kAcc][64 * 128];
  __nv_bfloat16 x[kAcc][128 * 64 + 64];
  uint4 ring[8 * kMmSlots * 128];  // [mixer warp][slot][2 KB]
  Page page[kPages];
  uint64_t plan_full[kPages], plan_empty[kPages];
  uint64_t x_full, x_empty, v_full, v_empty, o_full, o_empty, mma_done;
  uint32_t tmem_base;
  int abort;
};

using SmemBf16 = SmemT<false, false>;
using SmemFp8 = SmemT<true, false>;
using SmemMm = SmemT<false, true>;
static_assert(offsetof(SmemBf16, v) % 1024 == 0 && offsetof(SmemFp8, v) % 1024 == 0 && offsetof(SmemMm, v) == 0 &&
                  offsetof(SmemMm, x) % 1024 == 0,
              "V and X are 128-byte-swizzled operands");
static_assert(sizeof(SmemBf16) + 1024 <= 232448 && sizeof(SmemFp8) + 1024 <= 232448,
              "shared memory of one CTA (plus alignment slack) must fit the 227 KB opt-in limit");
static_assert(sizeof(SmemMm) <= 232448, "the tensor-core mixing's shared memory must fit the 227 KB opt-in limit");

struct Unit {
  int rb, hg, rg, I0, I1, Jmax;
};

__device__ __forceinline__ Unit decode(const Params& p, int k) {
  const int per = p.n_hg * p.n_rg;
  Unit u;
  u.rb = p.rb_hi - 1 - k / per;
  const int rest = k % per;
  u.hg = rest % p.n_hg;
  u.rg = rest / p.n_hg;
  // query blocks of the unit outside the output range are -1 (no entries, no rows written)
  if (p.B == 128) {
    u.I0 = u.rb;
    u.I1 = -1;
  } else {
    u.I0 = 2 * u.rb >= p.qb0 ? 2 * u.rb : -1;
    u.I1 = (2 * u.rb + 1 < p.qb1) ? 2 * u.rb + 1 : -1;
  }
  u.Jmax = u.I1 >= 0 ? u.I1 : u.I0;
  return u;
}

// The units of this CTA, longest first.  Grouped schedule (when a whole wave of `per` CTAs per
// group fits the grid): the CTAs of group g each own one (head group, request group) and walk
// the same row blocks n_rb - 1 - g - groups * t together, so the 16 or so CTAs that read a row
// block's map tiles read them at about the same time and the tiles are fetched from DRAM once and
// served from L2 to the others.  Otherwise: unit k = blockIdx.x + t * gridDim.x.
__device__ __forceinline__ int units_of_cta(const Params& p) {
  if (p.groups > 0) {
    const int g = blockIdx.x / p.per;
    return g < p.n_rb ? (p.n_rb - 1 - g) / p.groups + 1 : 0;
  }
  return (int)blockIdx.x < p.n_units ? (p.n_units - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
}
__device__ __forceinline__ Unit unit_at(const Params& p, int t) {
  if (p.groups > 0) {
    const int g = blockIdx.x / p.per, m = blockIdx.x % p.per;
    const int rb = p.rb_hi - 1 - (g + p.groups * t);
    // (rb, hg, rg) -> the index decode() maps back to the same unit
    return decode(p, (p.rb_hi - 1 - rb) * p.per + m);
  }
  return decode(p, (int)blockIdx.x + t * (int)gridDim.x);
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

template <typename S>
__device__ __forceinline__ void fail(S& s, const Params& p, uint32_t detail) {
  set_status(p.ws, MR_ERR_TIMEOUT, detail);
  s.abort = 1;
}

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

// ------------------------------------------------------------------------------------------------
// Planner warp: pages (one per sub-step, plus a marker after every unit and one at the end).  It
// waits only for page slots, never for the tensor core.
template <int G, bool F8, bool MM>
__device__ void planner(SmemT<F8, MM>& s, const Params& p) {
  using Page = typename SmemT<F8, MM>::Page;
  constexpr int kPages = SmemT<F8, MM>::kPages;
  const int lane = threadIdx.x & 31;
  uint32_t np = 0;    // pages written
  const int nparts = p.B / 64;
  bool ok = true;

  // lane 0 waits until page np's slot was released by every mixer warp
  auto claim = [&]() -> Page* {
    bool good = true;
    if (lane == 0 && np >= (uint32_t)kPages &&
        !mbar_wait_hint(&s.plan_empty[np % kPages], ((np / kPages) - 1) & 1, &s.abort, kTimeoutNs)) {
      fail(s, p, 0x101);
      good = false;
    }
    ok = __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
    return &s.page[np % kPages];
  };
  auto publish = [&]() {
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.plan_full[np % kPages]);
    ++np;
  };
  // Keep the CTAs of a schedule group together (they read the same map tiles, which then come
  // from DRAM once): hold page np back while the slowest member has consumed fewer than
  // np - kPages - kPaceSlack pages.  A hint only: after kPaceNs it goes ahead regardless, so a
  // member that is not resident (or finished) never blocks the others.
  auto pace = [&]() {
    if (p.groups <= 0 || p.per <= 1 || np <= (uint32_t)(kPages + kPaceSlack)) return;
    const uint32_t need = np - (uint32_t)(kPages + kPaceSlack);
    const int base = (int)(blockIdx.x / p.per) * p.per;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
      uint32_t lo = 0xffffffffu;
      for (int m = lane; m < p.per; m += 32) {
        const uint32_t v = ld_relaxed_gpu(p.progress + base + m);
        lo = v < lo ? v : lo;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const uint32_t w = __shfl_xor_sync(0xffffffffu, lo, o);
        lo = w < lo ? w : lo;
      }
      if (lo >= need || globaltimer_ns() - t0 > kPaceNs) break;
      __nanosleep(256);
    }
  };
  auto marker = [&](uint32_t flags) {
    Page* pg = claim();
    if (!ok) return;
    if (lane == 0) {
      pg->n = 0;
      pg->h = 0;
      pg->flags = flags;
    }
    publish();
  };
  const int nu = units_of_cta(p);
  for (int t = 0; t < nu && ok; ++t) {
    const Unit u = unit_at(p, t);
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
                              : 0ull;
      const uint64_t uni = m0 | m1;
      if (uni != 0) {
        for (int h = 0; h < nparts && ok; ++h) {
          pace();
          Page* pg = claim();
          if (!ok) break;
          // every lane writes the entries of its own sender heads, at their rank in the union
#pragma unroll
          for (int hs = 0; hs < 2; ++hs) {
            const int sh = lane + 32 * hs;
            if (!((uni >> sh) & 1ull)) continue;
            const int rank = __popcll((long long)(uni & ((1ull << sh) - 1ull)));
            auto& e = pg->e[rank];
#pragma unroll
            for (int pt = 0; pt < 2; ++pt) {
              uint32_t t = kNone;
              if (b[pt][hs]) {
                const int64_t tt = cur[pt][hs].first + cur[pt][hs].count;
                if (tt < p.capacity) {
                  t = (uint32_t)tt;
                  if (F8) {
                    const char* src = reinterpret_cast<const char*>(p.vals8 + tt * (int64_t)p.B * p.B) + 64 * p.B * h;
                    bulk_prefetch_l2(src, 64u * (uint32_t)p.B);
                  } else {
                    const char* src = reinterpret_cast<const char*>(p.vals + tt * (int64_t)p.B * p.B) +
                                      (p.B == 128 ? 16384 * h : 0);
                    bulk_prefetch_l2(src, p.B == 128 ? 16384u : 8192u);
                  }
                } else {
                  set_status(p.ws, MR_ERR_CAPACITY, 3u);  // the map overflowed: this tile was never stored
                }
              }
              e.t[pt] = t;
            }
#pragma unroll
            for (int g = 0; g < kAcc; ++g) e.w[g] = wv[hs][g];
            if constexpr (F8) {
              // the scales of the unit's four 32-row groups in panel h (rows 32 q .. of query block
              // I0 at block 128; two groups of I0 and two of I1 at block 64), rounded to bf16: the
              // relative error 2^-9 is small beside the e4m3 step of the values they scale
              uint32_t hb[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int pt = p.B == 128 ? 0 : q >> 1;
                const int rg = p.B == 128 ? q : q & 1;
                const uint32_t t = e.t[pt];
                const float sc = t != kNone ? __ldg(p.tile_scale + (size_t)t * fp8_scales_per_tile(p.B) +
                                                    rg * (p.B / 64) + (p.B == 128 ? h : 0))
                                            : 0.f;
                const __nv_bfloat16 b = __float2bfloat16_rn(sc);
                hb[q] = *reinterpret_cast<const uint16_t*>(&b);
              }
              e.sc[0] = hb[0] | (hb[1] << 16);
              e.sc[1] = hb[2] | (hb[3] << 16);
            }
          }
          if (lane == 0) {
            const uint32_t n = (uint32_t)__popcll((long long)uni);
            pg->n = n;
            pg->h = (uint32_t)h;
            pg->flags = 0u;
            if (n & 1u) pg->e[n].t[0] = pg->e[n].t[1] = kNone;  // mixers take entries in pairs
          }
          publish();
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
    marker(any_unit ? kUnitEnd : (kUnitEnd | kEmptyUnit));
  }
  if (ok) marker(kEnd);
}

// ------------------------------------------------------------------------------------------------
// Walks the sub-steps (unit, key block J, 64-key panel h) of this CTA in order.  Warp-collective.
struct SubWalker {
  int t, nu, J, h;
  Unit u;
  bool live;
  __device__ __forceinline__ void start(const Params& p) {
    t = 0;
    nu = units_of_cta(p);
    live = t < nu;
    if (live) u = unit_at(p, t);
    J = 0;
    h = -1;
  }
  // move to the next sub-step; false once the CTA has none left
  __device__ __forceinline__ bool next(const Params& p) {
    const int nparts = p.B / 64;
    while (live) {
      if (h >= 0 && h + 1 < nparts) {
        ++h;
        return true;
      }
      if (h >= 0) ++J;
      h = -1;
      for (; J <= u.Jmax; ++J) {
        const uint64_t m0 = head_mask(p, u.I0, J);
        const uint64_t m1 = (p.B == 64) ? head_mask(p, u.I1, J) : 0ull;
        if ((m0 | m1) != 0) {
          h = 0;
          return true;
        }
      }
      ++t;
      live = t < nu;
      if (live) u = unit_at(p, t);
      J = 0;
    }
    return false;
  }
};

template <int G, typename S>
__device__ void issue_v(S& s, const Params& p, const CUtensorMap* tmap_v, const Unit& u, int j0) {
  uint32_t bytes = 0;
  for (int a = 0; a < G * p.R; ++a)
    if (acc_valid(p, u, G, a)) bytes += 64 * 128 * 2;
  mbar_arrive_expect_tx(&s.v_full, bytes);
  for (int a = 0; a < G * p.R; ++a) {
    if (!acc_valid(p, u, G, a)) continue;
    const int r = u.hg * G + a / p.R, q = u.rg * p.R + a % p.R;
    const int g = r / p.v_group;
    int64_t row;
    if (p.v_pages) {
      // paged values: the 64 rows j0 .. j0 + 63 lie in one page (page_rows is a multiple of 64)
      const int64_t page = p.v_pages[(int64_t)q * p.pages_per_req + j0 / p.page_rows];
      row = (page * p.H_v + g) * p.page_rows + j0 % p.page_rows;
      if (page < 0 || (page * p.H_v + g + 1) * p.page_rows > p.v_rows) {
        set_status(p.ws, MR_ERR_DEVICE_CHECK, 6u);
        row = p.v_rows;
      }
    } else {
      const int64_t off = (p.v_req_off ? p.v_req_off[q] : (int64_t)q * p.v_req_stride) + (int64_t)g * p.v_head_stride;
      // a request's rows must start on a row of the tensor map and end inside the allocation; if
      // not, load from past the map's extent (TMA fills zeros) and record the bad offset
      row = off / 128 + j0;
      if (off < 0 || (off & 127) != 0 || off / 128 + (int64_t)p.L > p.v_rows) {
        set_status(p.ws, MR_ERR_DEVICE_CHECK, 5u);
        row = p.v_rows;
      }
    }
    tma_load_2d(&s.v[a][0], tmap_v, &s.v_full, 0, (int)row);
    tma_load_2d(&s.v[a][64 * 64], tmap_v, &s.v_full, 64, (int)row);
  }
}

// MMA warp: per sub-step, X (from the mixers) x V (loaded here one sub-step ahead) into the unit's
// accumulators; the next V load is issued once these MMAs have read the buffer.
template <int G, bool F8, bool MM>
__device__ void mma_issuer(SmemT<F8, MM>& s, const Params& p, const CUtensorMap* tmap_v) {
  const int lane = threadIdx.x & 31;
  const uint32_t idesc = idesc_bf16_f32(128, 128, false, true);
  const uint32_t tbase = s.tmem_base;
  uint32_t nsub = 0, nv = 0;
  int nunit = 0;
  bool ok = true;
  const int nparts = p.B / 64;
  SubWalker vw;  // the sub-step whose V is loaded next
  vw.start(p);
  if (vw.next(p)) {
    if (lane == 0) issue_v<G>(s, p, tmap_v, vw.u, vw.J * p.B + 64 * vw.h);
    ++nv;
  }
  const int nu = units_of_cta(p);
  for (; nunit < nu && ok; ++nunit) {
    const Unit u = unit_at(p, nunit);
    if (lane == 0 && nunit > 0 && !mbar_wait_hint(&s.o_empty, (nunit - 1) & 1, &s.abort, kTimeoutNs)) {
      fail(s, p, 0x201);
      ok = false;
    }
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (!ok) break;
    bool first = true;
    for (int J = 0; J <= u.Jmax && ok; ++J) {
      const uint64_t m0 = head_mask(p, u.I0, J);
      const uint64_t m1 = (p.B == 64) ? head_mask(p, u.I1, J) : 0ull;
      if ((m0 | m1) == 0) continue;
      for (int h = 0; h < nparts && ok; ++h) {
        if (lane == 0) {
          if (!mbar_wait_hint(&s.x_full, nsub & 1, &s.abort, kTimeoutNs) ||
              !mbar_wait_hint(&s.v_full, nsub & 1, &s.abort, kTimeoutNs)) {
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
        if (!ok) break;
        // the next sub-step's V, once these MMAs have read the buffer
        if (vw.next(p)) {
          if (lane == 0) {
            if (!mbar_wait_hint(&s.v_empty, (nsub - 1) & 1, &s.abort, kTimeoutNs)) {
              fail(s, p, 0x203);
              ok = false;
            } else {
              issue_v<G>(s, p, tmap_v, vw.u, vw.J * p.B + 64 * vw.h);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (ok) ++nv;
        }
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
  // drain: all MMAs issued by this thread complete before Tensor Memory is released, and the
  // last V load lands before shared memory is
  if (lane == 0) {
    mma_commit(&s.mma_done);
    const int never = 0;
    mbar_wait(&s.mma_done, 0, &never, kTimeoutNs);
    if (nv > 0) mbar_wait(&s.v_full, (nv - 1) & 1, &never, kTimeoutNs);
  }
  __syncwarp();
}

// ------------------------------------------------------------------------------------------------
// 16-byte global -> shared copy through L2 only, completed per thread by cp.async.wait_group
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// A stored word holds the e4m3 codes of keys (0, 2, 1, 3) of a group of four, all non-negative.
// Placing a code's 7 bits at bits 7..13 of a half gives exactly its value times 2^-8 (the exponent
// biases are 7 and 15; subnormals line up too), so a word splits into the half pairs of keys (0, 1)
// and (2, 3) with a mask and a shift each.
__device__ __forceinline__ __half2 e4m3_pair01(uint32_t w) {
  const uint32_t h = (w & 0x007F007Fu) << 7;
  return *reinterpret_cast<const __half2*>(&h);
}
__device__ __forceinline__ __half2 e4m3_pair23(uint32_t w) {
  const uint32_t h = (w >> 1) & 0x3F803F80u;
  return *reinterpret_cast<const __half2*>(&h);
}
// Four 8x8 b16 matrices from shared memory, transposed (thread t gets rows 2 (t % 4), + 1 of
// column t / 4 of each); lanes 8 m .. 8 m + 7 give the row addresses of matrix m.
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
// D (16 x 8, fp32) += A (16 x 16, bf16, row-major) * B (16 x 8, bf16, column-major), register operands.
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
               "{%0, %1, %2, %3};"
               : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// As cp_async16, issued only where `pred` holds (no branch).
__device__ __forceinline__ void cp_async16_if(uint32_t dst, const void* src, bool pred) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %2, 0;\n\t@p cp.async.cg.shared.global [%0], [%1], 16;\n\t}" ::"r"(dst),
      "l"(src), "r"((uint32_t)pred)
      : "memory");
}
template <int N>
struct Int {
  static constexpr int value = N;
};
// D (16 x 8, fp32) = A (16 x 16, bf16; rows 8 .. 15 zero) * B (16 x 8, bf16): the first k-step of a row.
__device__ __forceinline__ void mma_16816_z(float (&c)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %5}, {%7, %8}, "
               "{%9, %9, %9, %9};"
               : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
               : "r"(a0), "r"(0u), "r"(a2), "r"(b0), "r"(b1), "f"(0.f));
}
// Four 8x8 b16 matrices to shared memory in the MMA accumulator layout (thread t holds row t / 4,
// columns 2 (t % 4), + 1 of each); lanes 8 m .. 8 m + 7 give the row addresses of matrix m.
__device__ __forceinline__ void stsm_x4(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
  asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(r0), "r"(r1), "r"(r2),
               "r"(r3)
               : "memory");
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 b2 = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b2);
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr) : "memory");
  return v;
}

// Mixer warp w owns unit rows kRowsW * w .. + kRowsW - 1.  Thread (w, l) owns rows
// a_k = kRowsW * w + 4k + l/8 (k < kPieces) and, in each, the 16-byte chunk at physical position
// l % 8 of the 128-byte-swizzled
// panel row: eight consecutive keys 8 * ((l % 8) ^ (a_k % 8)).  X is written with the same
// swizzle, so the thread writes its chunks back to the positions it read them from.
// MM: mix on the tensor core with register operands (bf16 maps, block 128, at most 32 sender heads,
// 4 receiver heads of one request group); otherwise in fp32 / half FMAs on the CUDA cores.
template <int G, bool F8, bool MM>
__device__ void mixers(SmemT<F8, MM>& s, const Params& p) {
  using Page = typename SmemT<F8, MM>::Page;
  constexpr int kPages = SmemT<F8, MM>::kPages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int half = p.B == 64 ? (warp / (kMixWarps / 2)) : 0;  // 64-key blocks: which of the unit's two query blocks
  const uint32_t rowb = (uint32_t)(kRowsW * warp + (lane >> 3));
  const uint32_t my_off = (p.B == 64 ? (rowb & 63u) : rowb) * 128u + (uint32_t)(lane & 7) * 16u;  // bytes
  const uint32_t tile_bytes = (uint32_t)(p.B * p.B * 2);
  const char* vals = reinterpret_cast<const char*>(p.vals);
  // fp8 maps: thread (w, l) owns row rowb8 = 8 w + l / 4 of the unit and the 16-key piece l % 4 of
  // each 64-byte panel row; the scale of the 32-row x 64-key piece it falls in comes with the page entry
  const uint32_t rowb8 = (uint32_t)(kRowsW * warp + (lane >> 2));
  const uint32_t trow8 = p.B == 64 ? (rowb8 & 63u) : rowb8;
  const uint32_t my_off8 = trow8 * 64u + (uint32_t)(lane & 3) * 16u;
  const char* vals8 = reinterpret_cast<const char*>(p.vals8);
  const uint32_t tbase = s.tmem_base;
  const int tw = warp & 3;  // Tensor Memory lane quadrant of this warp

  // Fetch cursor (kQueue entry pairs ahead) and compute cursor over the page ring; a page of n
  // entries is taken as (n + 1) / 2 pairs (the planner pads odd pages with an empty entry).
  uint32_t pf = 0, ef = 0, nf = 0, hf = 0;  // page, pair, pairs in page, panel
  bool f_done = false;
  uint32_t pc = 0, ec = 0, nc = 0;
  const Page* cpg = &s.page[0];
  const Page* fpg = &s.page[0];
  uint32_t nsub = 0;
  int nunit = 0;

  auto wait_page = [&](uint32_t pg) -> bool {
    return mbar_wait_hint(&s.plan_full[pg % kPages], (pg / kPages) & 1, &s.abort, kTimeoutNs);
  };
  auto release_page = [&](uint32_t pg) {
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&s.plan_empty[pg % kPages]);
      if (warp == 0) st_relaxed_gpu(p.progress + blockIdx.x, pg + 1);
    }
  };
  // move the fetch cursor to the next page that lists panels (skipping markers); false on timeout
  auto fetch_seek = [&](uint32_t from) -> bool {
    for (uint32_t pg = from;; ++pg) {
      if (!wait_page(pg)) return false;
      const Page* P = &s.page[pg % kPages];
      const uint32_t n = P->n;
      if (n > 0) {
        pf = pg;
        fpg = P;
        ef = 0;
        nf = (n + 1) >> 1;
        hf = P->h;
        return true;
      }
      if (P->flags & kEnd) {
        f_done = true;
        return true;
      }
    }
  };
  // copy the next pair's pieces into ring slot `slot` (one cp.async group per pair, empty when
  // there is nothing to copy, so group counts stay aligned with pairs); the move to the
  // following page is taken lazily, at the next call
  const uint32_t ring0 = smem_u32(&s.ring[threadIdx.x]);
  constexpr int kPc = F8 ? kPieces8 : kPieces;
  constexpr uint32_t kPiece = kMixThreads * 16u, kEntry = kPc * kPiece, kSlot = 2u * kEntry;
  constexpr int kQueue = queue_of<F8>();
  auto fetch = [&](uint32_t slot) -> bool {
    bool good = true;
    if (!f_done && ef == nf) good = fetch_seek(pf + 1);
    if (good && !f_done && F8) {
      const uint32_t tt[2] = {fpg->e[2 * ef].t[half], fpg->e[2 * ef + 1].t[half]};
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        if (tt[j] == kNone) continue;
        const uint64_t t = tt[j];
        cp_async16(ring0 + slot * kSlot + j * kEntry,
                   vals8 + (t * (uint64_t)(p.B * p.B) + hf * 64u * (uint32_t)p.B + my_off8));
      }
      ++ef;
    } else if (good && !f_done) {
      const uint32_t t0 = fpg->e[2 * ef].t[half], t1 = fpg->e[2 * ef + 1].t[half];
      const uint32_t dst = ring0 + slot * kSlot;
      const uint32_t panel = hf * 16384u + my_off;
      if (t0 != kNone) {
        const char* src = vals + ((uint64_t)t0 * tile_bytes + panel);
#pragma unroll
        for (int k = 0; k < kPieces; ++k) cp_async16(dst + k * kPiece, src + 512 * k);
      }
      if (t1 != kNone) {
        const char* src = vals + ((uint64_t)t1 * tile_bytes + panel);
#pragma unroll
        for (int k = 0; k < kPieces; ++k) cp_async16(dst + kEntry + k * kPiece, src + 512 * k);
      }
      ++ef;
    }
    cp_async_commit();
    return good;
  };

  constexpr int kW = 4 * kPieces;  // packed bf16 pairs per thread per panel
  float2 acc[G][kW];               // fp32 accumulators for columns (2e, 2e + 1) of the thread's chunks
  __half2 acch[G][8];              // fp8 maps: half accumulators of the thread's 16 keys (x 2^14)
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < kW; ++e) {
      acc[g][e] = make_float2(0.f, 0.f);
      acch[g][e] = __float2half2_rn(0.f);
    }

  // fp8 entry: acch[g] += (W[r_g, s] * scale * 2^14) * (the thread's 16 e4m3 values)
  auto mix_entry8 = [&](const auto& E, uint32_t data) {
    const uint32_t scw = E.sc[rowb8 >> 6];
    const float sc = __uint_as_float((rowb8 & 32u) ? (scw & 0xffff0000u) : (scw << 16)) * (kF8Pre * kF8Decode);
    __half2 w2[G];
#pragma unroll
    for (int g = 0; g < G; ++g) w2[g] = __float2half2_rn(E.w[g] * sc);
    const uint4 d = lds128(data);
    const uint32_t wd[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __half2 lo = e4m3_pair01(wd[e]), hi = e4m3_pair23(wd[e]);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        acch[g][2 * e] = __hfma2(w2[g], lo, acch[g][2 * e]);
        acch[g][2 * e + 1] = __hfma2(w2[g], hi, acch[g][2 * e + 1]);
      }
    }
  };

  // one entry: acc[g] += W[r_g, s] * (this thread's 16 values of the sender head's panel)
  auto mix_entry = [&](const auto& E, uint32_t data) {
    const float4 wf = *reinterpret_cast<const float4*>(&E.w[0]);
    const float w[4] = {wf.x, wf.y, wf.z, wf.w};
    float2 w2[G];
#pragma unroll
    for (int g = 0; g < G; ++g) w2[g] = make_float2(w[g], w[g]);
#pragma unroll
    for (int k = 0; k < kPieces; ++k) {
      const uint4 d = lds128(data + k * kPiece);
      const uint32_t wd[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = 4 * k + e;
        // bf16 pair -> fp32 pair: the low half is the lower column (measured: a shift here beats a
        // byte permute, which loads the integer pipe with both halves)
        const float2 v = make_float2(__uint_as_float(wd[e] << 16), __uint_as_float(wd[e] & 0xffff0000u));
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g][c] = __ffma2_rn(w2[g], v, acc[g][c]);
      }
    }
  };

  // X of one sub-step, once the previous sub-step's MMAs have read the buffer
  auto hand_x = [&]() -> bool {
    if (nsub > 0 && !mbar_wait_hint(&s.x_empty, (nsub - 1) & 1, &s.abort, kTimeoutNs)) return false;
#pragma unroll
    for (int g = 0; g < (F8 ? G : 0); ++g) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {  // the thread's two 8-key chunks of X row rowb8
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 a = __half22float2(acch[g][4 * c + e]);
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(a.x, a.y);
          pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
          acch[g][4 * c + e] = __float2half2_rn(0.f);
        }
        const uint32_t lc = 2u * (uint32_t)(lane & 3) + (uint32_t)c;
        char* xb = reinterpret_cast<char*>(&s.x[g][0]) + rowb8 * 128 + ((lc ^ ((rowb8 + g) & 7u)) << 4);
        *reinterpret_cast<uint4*>(xb) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
#pragma unroll
    for (int g = 0; g < (F8 ? 0 : G); ++g) {
#pragma unroll
      for (int k = 0; k < kPieces; ++k) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 a = acc[g][4 * k + e];
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(a.x, a.y);
          pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
          acc[g][4 * k + e] = make_float2(0.f, 0.f);
        }
        // the chunk read from physical position l % 8 of a panel row (phase row % 8) goes to the
        // same logical chunk of X row `row` (phase (row + g) % 8)
        const uint32_t row = rowb + 4 * k;
        char* xb = reinterpret_cast<char*>(&s.x[g][0]) + row * 128 + (((lane & 7) ^ (row & 7u) ^ ((row + g) & 7u)) << 4);
        *reinterpret_cast<uint4*>(xb) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.x_full);
    ++nsub;
    return true;
  };
  // the unit's accumulators -> bf16 -> O (warp w stores accumulators w / 4 + 2 i of its 32 rows)
  auto epilogue = [&](bool any) -> bool {
    if (!mbar_wait_hint(&s.o_full, nunit & 1, &s.abort, kTimeoutNs)) return false;
    tc_fence_after();
    const Unit u = unit_at(p, nunit);
    const int row = 32 * tw + lane;
    const int i = u.rb * 128 + row;
    const int qblk = p.B == 128 ? u.rb : 2 * u.rb + (row >> 6);
    const bool row_out = i < p.L && qblk >= p.qb0 && qblk < p.qb1;  // rows outside the range stay as they are
    const float osc = F8 ? 1.f / kF8Pre : 1.f;                       // fp8 maps were mixed x 2^14
#pragma unroll 1
    for (int a = warp >> 2; a < G * p.R; a += (MM ? 8 : kMixWarps) / 4) {
      const bool valid = acc_valid(p, u, G, a);
      const int r = u.hg * G + a / p.R, q = u.rg * p.R + a % p.R;
      __nv_bfloat16* orow = p.O + (((size_t)q * p.H_r + r) * p.L + i) * 128;
#pragma unroll 1
      for (int cc = 0; cc < 8; ++cc) {
        uint32_t v[16];
        tmem_ld16(tbase + ((uint32_t)(32 * tw) << 16) + 128 * a + 16 * cc, v);
        tmem_wait_ld();
        if (valid && row_out && checked(p.ws, q < p.n_req && r < p.H_r && i < p.L, 0xC31)) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = any ? __uint_as_float(v[8 * c + 2 * e]) * osc : 0.f;
              const float x1 = any ? __uint_as_float(v[8 * c + 2 * e + 1]) * osc : 0.f;
              const __nv_bfloat162 b2 = __floats2bfloat162_rn(x0, x1);
              pk[e] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            *reinterpret_cast<uint4*>(orow + 16 * cc + 8 * c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.o_empty);
    ++nunit;
    return true;
  };
  // process marker pages from pc on until a page that lists panels (or the end); false = stop
  auto compute_seek = [&](bool& stop) -> bool {
    for (;;) {
      if (!wait_page(pc)) return false;
      const Page* P = &s.page[pc % kPages];
      const uint32_t n = P->n, fl = P->flags;
      if (n > 0) {
        cpg = P;
        ec = 0;
        nc = (n + 1) >> 1;
        return true;
      }
      if (fl & kUnitEnd) {
        if (!epilogue(!(fl & kEmptyUnit))) return false;
      }
      if (fl & kEnd) {
        stop = true;
        return true;
      }
      release_page(pc);
      ++pc;
    }
  };

  if (MM) {
    // ---- head mixing as a tensor-core contraction over sender heads ---------------------------
    // X_g[i, j] = sum_s W[g, s] A_s[i, j] is, for each unit row i, a product of the page's weights
    // (A operand: 16 rows, the first G of them receiver heads; 16 sender heads per k-step) and the
    // sender heads' values in that row (B operand: 16 heads x 8 keys per n-tile, through a
    // transposed matrix load), accumulated in fp32 registers: no Tensor Memory (all of it holds the
    // Ã·V accumulators) and no per-thread accumulator arrays.  8 mixer warps; warp w owns unit rows
    // 16 w .. 16 w + 15.  A step is one row and one k-step: the row's 128 bytes in each of 16
    // sender heads, copied by the warp into a private 2 KB slot of a kMmSlots-deep ring, so the warp waits
    // on its own copies only.  Head e's row sits at e * 128 with the map's physical chunk q at
    // q ^ (e % 8), so the eight rows of each transposed load hit eight different bank groups.
    constexpr uint32_t kD = kMmSlots, kRows = 16;
    // rows 0..kHold are computed before the wait for X (measured at 32K tokens with 200 registers:
    // kHold 0 54.0 ms, 1 54.9, 2 55.9, 3 58.9)
    constexpr uint32_t kHold = 0;
    static_assert(!MM || sizeof(s.ring) == 8 * kD * 2048, "8 warps x kD slots of 2 KB");
    static_assert(!MM || G == 4, "the first four rows of the product are the receiver heads");
    char* wring_g = reinterpret_cast<char*>(&s.ring[0]) + (uint32_t)warp * (kD * 2048u);
    const uint32_t wring = smem_u32(wring_g);
    for (uint32_t off = (uint32_t)lane * 16u; off < kD * 2048u; off += 512u)
      *reinterpret_cast<uint4*>(wring_g + off) = make_uint4(0u, 0u, 0u, 0u);  // unlisted heads: weight 0, finite values
    __syncwarp();
    const uint32_t q = (uint32_t)lane & 7u, lh = (uint32_t)lane >> 3;
    // copies: lane (lh, q) moves chunk q of heads 4 jj + lh (jj < 4); slot offsets for even and odd
    // jj, + 1024 for jj >= 2
    const uint32_t dst_even = lh * 128u + ((q ^ lh) << 4), dst_odd = 512u + lh * 128u + ((q ^ (4u + lh)) << 4);
    // transposed loads: lane 8 m + r gives row r of matrix m, i.e. head 8 (m % 2) + r and logical
    // chunk 2 i + m / 2 of the row, stored at (2 i + m / 2) ^ (row % 8) ^ r
    const uint32_t ld_row = (8u * (lh & 1u) + q) * 128u, ld_z = (lh >> 1) ^ q;
    // matrix stores of a finished row: lane 8 m + r gives row r of n-tile 4 k + m.  Rows r < 4 are
    // the receiver heads' X rows (swizzle phase (R + r) % 8); rows 4..7 of the product are zero and
    // go to the 128-byte gap after X buffer r - 4, at the phases (R + r) % 8 the receivers leave free, so
    // the eight rows of each matrix fall in eight different bank groups
    const bool st_real = q < 4u;
    const uint32_t st_base = smem_u32(st_real ? &s.x[q & 3u][0] : &s.x[q & 3u][128 * 64]);  // gap after buffer r - 4
    const uint32_t st_rowmask = st_real ? 0xffffffffu : 0u;
    const uint32_t st_u0 = lh << 4;
    auto store_row = [&](uint32_t row, const uint32_t (&w)[8]) {
      const uint32_t R = kRows * (uint32_t)warp + row;
      const uint32_t base = st_base + ((R * 128u) & st_rowmask);
      const uint32_t u = st_u0 ^ (((R + q) & 7u) << 4);
      stsm_x4(base | u, w[0], w[1], w[2], w[3]);
      stsm_x4(base | (u ^ 64u), w[4], w[5], w[6], w[7]);
    };

    // fetch cursor: page, step within it (row = step >> f_sh, k-step = step & f_sh), the lane's tiles
    uint32_t f_pg = 0, f_s = 0, f_steps = 0, f_sh = 0;
    bool f_end = false;
    const char* f_src = vals;  // chunk q of the warp's first row in the page's panel of tile 0
    uint32_t tl0[4], tl1[4];   // tiles of heads 4 jj + lh and 16 + 4 jj + lh (kNone: no copy)
    auto f_seek = [&](uint32_t from) -> bool {
      for (uint32_t pg = from;; ++pg) {
        if (!wait_page(pg)) return false;
        const Page* P = &s.page[pg % kPages];
        const uint32_t n = P->n;
        if (n > 0) {
          f_pg = pg;
          f_s = 0;
          f_sh = n > 16u ? 1u : 0u;
          f_steps = kRows << f_sh;
          f_src = vals + (P->h * 16384u + (uint32_t)warp * (kRows * 128u) + q * 16u);
#pragma unroll
          for (uint32_t jj = 0; jj < 4; ++jj) {
            const uint32_t e0 = 4u * jj + lh, e1 = 16u + e0;
            tl0[jj] = e0 < n ? P->e[e0].t[0] : kNone;
            tl1[jj] = e1 < n ? P->e[e1].t[0] : kNone;
          }
          return true;
        }
        if (P->flags & kEnd) {
          f_end = true;
          return true;
        }
      }
    };
    // copy the next step into `slot`: one cp.async group per step, empty at the end
    auto fetch_step = [&](uint32_t slot) -> bool {
      bool ok = true;
      if (!f_end && f_s == f_steps) ok = f_seek(f_pg + 1);
      if (ok && !f_end) {
        const uint32_t kt = f_s & f_sh;
        const char* src = f_src + (f_s >> f_sh) * 128u;
        const uint32_t d = wring + slot * 2048u;
#pragma unroll
        for (uint32_t jj = 0; jj < 4; ++jj) {
          const uint32_t t = kt ? tl1[jj] : tl0[jj];
          cp_async16_if(d + ((jj & 1u) ? dst_odd : dst_even) + (jj >> 1) * 1024u, src + (uint64_t)t * 32768u, t != kNone);
        }
        ++f_s;
      }
      cp_async_commit();
      return ok;
    };
    // A fragments of the compute page: receiver lane / 4 (zero beyond G), heads 16 kt + 2 (lane % 4)
    // + {0, 1} (first register) and + 8 + {0, 1} (second); rows 8 .. 15 of A are zero
    uint32_t afr[2][2];
    uint32_t c_nkt = 1;
    auto build_a = [&]() {
      const uint32_t n = cpg->n;
      c_nkt = n > 16u ? 2u : 1u;
      const int g = lane >> 2;
#pragma unroll
      for (int kt = 0; kt < 2; ++kt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint32_t e0 = 16u * kt + 8u * hh + 2u * ((uint32_t)lane & 3u);
          float w0 = 0.f, w1 = 0.f;
          if (g < G) {
            if (e0 < n && cpg->e[e0].t[0] != kNone) w0 = cpg->e[e0].w[g];
            if (e0 + 1u < n && cpg->e[e0 + 1u].t[0] != kNone) w1 = cpg->e[e0 + 1u].w[g];
          }
          afr[kt][hh] = pack_bf16x2(w0, w1);
        }
    };
    bool stop = false;
    bool good = f_seek(0) && compute_seek(stop);
    if (good && !stop) build_a();
    for (uint32_t u = 0; u < kD; ++u)
      if (good && !stop) good = fetch_step(u);
    uint32_t slot = 0;
    // copy step (row, KT) of the compute page into `slot` (the fetch cursor's tiles are that page's)
    auto fetch_static = [&](uint32_t slot_, uint32_t row, auto KT) {
      const char* src = f_src + row * 128u;
      const uint32_t d = wring + slot_ * 2048u;
#pragma unroll
      for (uint32_t jj = 0; jj < 4; ++jj) {
        const uint32_t t = decltype(KT)::value ? tl1[jj] : tl0[jj];
        cp_async16_if(d + ((jj & 1u) ? dst_odd : dst_even) + (jj >> 1) * 1024u, src + (uint64_t)t * 32768u, t != kNone);
      }
      cp_async_commit();
    };
    // one k-step of a row: wait for its slot, load it as B fragments, multiply, refill the slot with
    // the step kD ahead: (row + (KT + kD) / NKT, (KT + kD) % NKT) of this page, or (TAIL) the
    // cursor's next step
    auto kstep = [&](uint32_t row, float (&acc)[8][4], auto KT, auto NKT, auto TAIL) {
      cp_async_wait<kD - 1>();  // this lane's copies of the oldest step have landed
      __syncwarp();             // ... and every other lane's
      const uint32_t lrow = wring + slot * 2048u + ld_row;
      const uint32_t z = (ld_z ^ (row & 7u)) << 4;
      uint32_t b[4][4];  // [load i][matrix]: n-tiles 2 i and 2 i + 1, heads 0..7 and 8..15 of the k-step
#pragma unroll
      for (uint32_t i = 0; i < 4; ++i) ldsm_x4_trans(b[i], lrow | (z ^ (32u * i)));
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        if (decltype(KT)::value == 0)
          mma_16816_z(acc[nt], afr[0][0], afr[0][1], b[nt >> 1][2 * (nt & 1)], b[nt >> 1][2 * (nt & 1) + 1]);
        else
          mma_16816(acc[nt], afr[1][0], 0u, afr[1][1], 0u, b[nt >> 1][2 * (nt & 1)], b[nt >> 1][2 * (nt & 1) + 1]);
      }
      __syncwarp();  // every lane's loads of the slot are in the MMAs above before any lane refills it
      if constexpr (decltype(TAIL)::value) {
        if (!fetch_step(slot)) good = false;
      } else {
        constexpr int kN = decltype(NKT)::value, kAhead = decltype(KT)::value + (int)kD;
        fetch_static(slot, row + (uint32_t)(kAhead / kN), Int<kAhead % kN>{});
      }
      slot = slot + 1u == kD ? 0u : slot + 1u;
    };
    // a whole row: its k-steps, then the receivers' X values packed to bf16
    auto row_x = [&](uint32_t row, uint32_t (&pk)[8], auto NKT, auto TAIL) {
      float acc[8][4];
      kstep(row, acc, Int<0>{}, NKT, TAIL);
      if constexpr (decltype(NKT)::value == 2) kstep(row, acc, Int<1>{}, NKT, TAIL);
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) pk[nt] = pack_bf16x2(acc[nt][0], acc[nt][1]);
    };
    // the warp's 16 rows of one sub-step; rows 0..kHold are held until X is free.  On entry the fetch
    // cursor has copied the page's first kD steps.  Rows before kTail fetch kD steps ahead within
    // the page; the rest fetch through the cursor, which resumes at the first step they leave (the
    // page's last steps, then the next page's first kD).
    auto sub_step = [&](auto NKT) -> bool {
      constexpr uint32_t kN = decltype(NKT)::value;
      constexpr uint32_t kTail = kRows - (kD + kN - 1) / kN;
      f_s = kTail * kN + kD;
      uint32_t held[kHold + 1][8];
#pragma unroll
      for (uint32_t r = 0; r <= kHold; ++r) row_x(r, held[r], NKT, Int<0>{});
      // X is free once the previous sub-step's MMAs have read it
      bool ok = true;
      if (lane == 0 && nsub > 0) ok = mbar_wait_hint(&s.x_empty, (nsub - 1) & 1, &s.abort, kTimeoutNs);
      if (__shfl_sync(0xffffffffu, ok ? 1 : 0, 0) == 0) return false;
#pragma unroll
      for (uint32_t r = 0; r <= kHold; ++r) store_row(r, held[r]);
      uint32_t pk[8];
#pragma unroll 1
      for (uint32_t row = kHold + 1; row < kTail; ++row) {
        row_x(row, pk, NKT, Int<0>{});
        store_row(row, pk);
      }
#pragma unroll 1
      for (uint32_t row = kTail; row < kRows; ++row) {
        row_x(row, pk, NKT, Int<1>{});
        store_row(row, pk);
      }
      return true;
    };
    while (good && !stop) {
      const bool ok = c_nkt == 2 ? sub_step(Int<2>{}) : sub_step(Int<1>{});
      if (!ok || !good) {
        good = false;
        break;
      }
      // end of the sub-step: X to the tensor core, release the page, run any markers
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.x_full);
      ++nsub;
      release_page(pc);
      ++pc;
      if (!compute_seek(stop)) {
        good = false;
        break;
      }
      if (!stop) build_a();
    }
    cp_async_wait<0>();  // no copy may land after the CTA releases its shared memory
    if (!good) fail(s, p, 0x302);
    return;
  }

  bool stop = false;
  bool good = fetch_seek(0) && compute_seek(stop);
  for (uint32_t u = 0; u < (uint32_t)kQueue; ++u)
    if (good && !stop) good = fetch(u);
  uint32_t slot = 0;
  while (good && !stop) {
    cp_async_wait<kQueue - 1>();  // this thread's copies of the oldest pair have landed
    const uint32_t data = ring0 + slot * kSlot;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const auto& E = cpg->e[2 * ec + j];
      if (E.t[half] != kNone) {
        if constexpr (F8)
          mix_entry8(E, data + j * kEntry);
        else
          mix_entry(E, data + j * kEntry);
      }
    }
    if (++ec == nc) {
      // end of the sub-step: hand X to the tensor core, release the page, run any markers
      if (!hand_x()) {
        good = false;
        break;
      }
      release_page(pc);
      ++pc;
      if (!compute_seek(stop)) {
        good = false;
        break;
      }
    }
    // refill this slot kQueue pairs ahead
    if (!stop) good = fetch(slot);
    slot = (slot + 1 == (uint32_t)kQueue) ? 0u : slot + 1;
  }
  cp_async_wait<0>();  // no copy may land after the CTA releases its shared memory
  if (!good) fail(s, p, 0x301);
}

// Mixer warps of an instantiation: 16 on the CUDA-core mixing path, 8 on the tensor-core one.
template <bool MM>
struct Roles {
  static constexpr int kMix = MM ? 8 : kMixWarps;
  static constexpr int kPlan = kMix, kMma = kMix + 1;
  // tensor-core mixing: two idle warps complete a third warpgroup with the planner and the MMA
  // warp, which gives up registers (setmaxnreg) to the mixers' two warpgroups
  static constexpr int kThreadsK = MM ? 384 : (kMix + 2) * 32;
};
constexpr int kMmLaunchRegs = 168, kMmRegsControl = 104, kMmRegsMix = 200;
static_assert(kMmRegsControl + 2 * kMmRegsMix == 3 * kMmLaunchRegs, "register split of the tensor-core mixing launch");

template <int G, bool F8, bool MM>
__global__ void __launch_bounds__(Roles<MM>::kThreadsK, 1) k_retrieve_tc(const __grid_constant__ CUtensorMap tmap_v, Params p) {
  constexpr int kMixWarps = Roles<MM>::kMix, kPlanWarp = Roles<MM>::kPlan, kMmaWarp = Roles<MM>::kMma;
  extern __shared__ unsigned char smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  if constexpr (MM) {
    // no slack to align in this layout: the dynamic shared memory must start on a 1024-byte boundary
    if (pad != 0) {
      if (threadIdx.x == 0) set_status(p.ws, MR_ERR_DEVICE_CHECK, 9u);
      return;
    }
  }
  SmemT<F8, MM>& s = *reinterpret_cast<SmemT<F8, MM>*>(smem_raw + pad);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int i = 0; i < SmemT<F8, MM>::kPages; ++i) {
      mbar_init(&s.plan_full[i], 1);
      mbar_init(&s.plan_empty[i], kMixWarps);
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
  if constexpr (MM) {
    // every warp of the control warpgroup gives its registers back before any role starts, so
    // the mixers' increase never waits on a role
    if (warp < kMixWarps) {
      regs_inc<kMmRegsMix>();
      mixers<G, F8, MM>(s, p);
    } else {
      regs_dec<kMmRegsControl>();
      if (warp == kPlanWarp)
        planner<G, F8, MM>(s, p);
      else if (warp == kMmaWarp)
        mma_issuer<G, F8, MM>(s, p, &tmap_v);
    }
  } else {
    if (warp < kMixWarps)
      mixers<G, F8, MM>(s, p);
    else if (warp == kPlanWarp)
      planner<G, F8, MM>(s, p);
    else
      mma_issuer<G, F8, MM>(s, p, &tmap_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(s.tmem_base, 512);
}

template <int G, bool F8, bool MM = false>
cudaError_t launch_g(const RetrieveArgs& a, const Params& p, const CUtensorMap& tm, int grid, cudaStream_t st) {
  const size_t smem = sizeof(SmemT<F8, MM>) + (MM ? 0 : 1024);
  cudaError_t e;
  if (MM) {
    // the register split assumes the launch allocation it was sized for
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, k_retrieve_tc<G, F8, MM>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kMmLaunchRegs) return cudaErrorInvalidConfiguration;
  }
  e = cudaFuncSetAttribute(k_retrieve_tc<G, F8, MM>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  ProfScope ps(kKRetrieveTc, st);
  k_retrieve_tc<G, F8, MM><<<grid, Roles<MM>::kThreadsK, smem, st>>>(tm, p);
  return cudaGetLastError();
}

template <bool F8>
cudaError_t launch_any(const RetrieveArgs& a, const Params& p, const CUtensorMap& tm, int grid, int G) {
  // bf16 maps of 128-key blocks with at most 32 sender heads, 4 receiver heads per CTA: mixing
  // on the tensor core
  if (!F8 && G == 4 && p.B == 128 && p.H_s <= 32) return launch_g<4, false, true>(a, p, tm, grid, a.stream);
  if (G == 4) return launch_g<4, F8>(a, p, tm, grid, a.stream);
  if (G == 2) return launch_g<2, F8>(a, p, tm, grid, a.stream);
  return launch_g<1, F8>(a, p, tm, grid, a.stream);
}

}  // namespace

bool tc_retrieve_supported(const RetrieveArgs& a) {
  return a.dt == MR_BF16 && (a.map.val_dtype == MR_BF16 || a.map.val_dtype == MR_FP8_E4M3) && a.d_v == 128 && (a.map.block == 64 || a.map.block == 128) && a.map.H_s <= 64 &&
         a.map.capacity_tiles < (int64_t)kNone && (a.v_pages != nullptr || a.v_head_stride % 128 == 0) &&
         (a.v_pages != nullptr || a.v_req_off != nullptr || a.v_req_stride % 128 == 0) &&
         a.v_elems / 128 < ((int64_t)1 << 31) - 1;
}

cudaError_t tc_retrieve(const RetrieveArgs& a) {
  Params p;
  p.kept_bits = a.map.kept_bits;
  p.row_ptr = a.map.row_ptr;
  p.vals = (const __nv_bfloat16*)a.map.vals;
  p.vals8 = (const uint8_t*)a.map.vals;
  p.tile_scale = a.map.tile_scale;
  p.capacity = a.map.capacity_tiles;
  p.W = a.W;
  p.O = (__nv_bfloat16*)a.O;
  p.v_req_off = a.v_req_off;
  p.v_req_stride = a.v_req_stride;
  p.v_head_stride = a.v_head_stride;
  p.v_rows = a.v_elems / 128;
  p.v_group = a.v_group;
  p.H_v = a.H_r / a.v_group;
  p.v_pages = a.v_pages;
  p.page_rows = a.page_rows;
  p.pages_per_req = a.pages_per_req;
  p.H_s = a.map.H_s;
  p.H_r = a.H_r;
  p.L = a.map.L;
  p.B = a.map.block;
  p.nqb = a.map.L / a.map.block;
  p.nkw = (p.nqb + 31) / 32;
  p.n_req = a.n_req;
  p.qb0 = a.qb0;
  p.qb1 = a.qb1;
  int G = 4;
  if (a.n_req >= 4)
    G = 1;
  else if (a.n_req >= 2)
    G = 2;
  p.R = kAcc / G;
  p.n_hg = (a.H_r + G - 1) / G;
  p.n_rg = (a.n_req + p.R - 1) / p.R;
  // 128-row blocks holding the output query blocks
  const int rb_lo = p.B == 128 ? a.qb0 : a.qb0 / 2;
  p.rb_hi = p.B == 128 ? a.qb1 : (a.qb1 + 1) / 2;
  p.n_rb = p.rb_hi - rb_lo;
  p.n_units = p.n_rb * p.n_hg * p.n_rg;
  p.per = p.n_hg * p.n_rg;
  p.ws = a.ws;
  p.progress = reinterpret_cast<uint32_t*>(reinterpret_cast<char*>(a.ws) + kWsHeaderBytes);
  // V viewed as rows of 128 bf16 spanning exactly the caller's allocation: rows past it read as
  // zeros, and offsets are checked against it on the device
  CUtensorMap tm;
  if (!make_tmap_bf16_2d(&tm, a.V, 128, (uint64_t)p.v_rows, 256, 64, 64)) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int grid;
  if (p.per <= sms && sms <= kMaxProgressCtas) {
    p.groups = sms / p.per < p.n_rb ? sms / p.per : p.n_rb;
    grid = p.groups * p.per;
  } else {
    p.groups = 0;
    grid = p.n_units < sms ? p.n_units : sms;
    if (grid > kMaxProgressCtas) grid = kMaxProgressCtas;  // one progress counter per CTA
  }
  if (a.map.val_dtype == MR_FP8_E4M3) return launch_any<true>(a, p, tm, grid, G);
  return launch_any<false>(a, p, tm, grid, G);
}

}  // namespace mr
