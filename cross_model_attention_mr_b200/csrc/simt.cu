// CUDA-core (SIMT) kernels for compression, retrieval and dense attention.
//
// These run the fp32 workloads (tensor cores would need tf32, which the fp32 tolerance rules
// out) and give a plain, easily checked CUDA path for every shape.  Each CTA owns one unit of
// the method's parallel work: a (head, query block) row of the map for compression, a (query
// block, receiver head, request) output tile for retrieval, and a (sequence tile, head) for dense
// attention.  Work units with more causal tiles are scheduled first (larger query blocks first).
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"
#include "profile.h"

namespace mr {
namespace {

constexpr int kThreads = 256;

template <typename T, int ROWS, int D>
__device__ __forceinline__ void load_rows(float* dst, const T* __restrict__ src, int valid_rows) {
  for (int e = threadIdx.x; e < ROWS * D; e += kThreads) {
    const int r = e / D, c = e - (e / D) * D;
    dst[r * (D + 1) + c] = (r < valid_rows) ? to_f32(src[(size_t)r * D + c]) : 0.f;
  }
}

// Scores of a ROWS x COLS tile: thread (ty = tid / 16, tx = tid % 16) owns rows ty + 16a and
// columns tx + 16b.
template <int ROWS, int COLS, int D>
__device__ __forceinline__ void tile_dot(const float* Qs, const float* Ks, float (&S)[ROWS / 16][COLS / 16]) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int a = 0; a < ROWS / 16; ++a)
#pragma unroll
    for (int b = 0; b < COLS / 16; ++b) S[a][b] = 0.f;
#pragma unroll 4
  for (int k = 0; k < D; ++k) {
    float qv[ROWS / 16], kv[COLS / 16];
#pragma unroll
    for (int a = 0; a < ROWS / 16; ++a) qv[a] = Qs[(ty + 16 * a) * (D + 1) + k];
#pragma unroll
    for (int b = 0; b < COLS / 16; ++b) kv[b] = Ks[(tx + 16 * b) * (D + 1) + k];
#pragma unroll
    for (int a = 0; a < ROWS / 16; ++a)
#pragma unroll
      for (int b = 0; b < COLS / 16; ++b) S[a][b] = fmaf(qv[a], kv[b], S[a][b]);
  }
}

__device__ __forceinline__ float group16_max(float v) {
#pragma unroll
  for (int o = 8; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float group16_sum(float v) {
#pragma unroll
  for (int o = 8; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------------------------
// Compression, part 1: per (head h, query block I) row statistics, block masses, top-p selection.
// Three sweeps over key blocks J <= I: row maxima, row sums, then block masses of the normalised
// probabilities.  Selection ranks blocks by the 64-bit key (mass bits, ~J) (larger mass first,
// smaller J on ties) and takes the shortest prefix whose fp64 cumulative mass reaches p.
// ---------------------------------------------------------------------------------------------
template <typename T, int BLK, int D>
__global__ void __launch_bounds__(kThreads) k_compress_stats(
    const T* __restrict__ Q, const T* __restrict__ K, int H, int L, float scale, float p, Bias bias,
    float* __restrict__ lse_ws, int* __restrict__ count_ws, uint32_t* __restrict__ kept_bits,
    float* __restrict__ kept_mass, float* __restrict__ mass_out, float* __restrict__ lse_out, int qb_hi,
    int renorm) {
  extern __shared__ float smem[];
  float* Qs = smem;
  float* Ks = Qs + BLK * (D + 1);
  __shared__ float row_m[BLK];
  __shared__ float row_l[BLK];
  __shared__ float mass_s[256];
  __shared__ int sorted_s[256];
  __shared__ uint32_t bits_s[8];
  __shared__ float red[kThreads / 32];
  __shared__ int kstar_s;

  const int nqb = L / BLK, nkb = nqb, nkw = (nkb + 31) / 32;
  const int I = qb_hi - 1 - (int)(blockIdx.x / H);  // query blocks qb_hi - 1, qb_hi - 2, ...
  const int h = (int)(blockIdx.x % H);
  const int u = h * nqb + I;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  constexpr int R = BLK / 16;

  load_rows<T, BLK, D>(Qs, Q + ((size_t)h * L + (size_t)I * BLK) * D, BLK);
  for (int r = tid; r < BLK; r += kThreads) {
    row_m[r] = -INFINITY;
    row_l[r] = 0.f;
  }
  for (int J = tid; J < 256; J += kThreads) mass_s[J] = 0.f;

  for (int pass = 0; pass < 3; ++pass) {
    for (int J = 0; J <= I; ++J) {
      __syncthreads();
      load_rows<T, BLK, D>(Ks, K + ((size_t)h * L + (size_t)J * BLK) * D, BLK);
      __syncthreads();
      float S[R][R];
      tile_dot<BLK, BLK, D>(Qs, Ks, S);
      float part = 0.f;
#pragma unroll
      for (int a = 0; a < R; ++a) {
        const int r = ty + 16 * a;
        const int i = I * BLK + r;
        const float ref = row_m[r];
        float acc = (pass == 0) ? -INFINITY : 0.f;
#pragma unroll
        for (int b = 0; b < R; ++b) {
          const int j = J * BLK + tx + 16 * b;
          if (j <= i) {
            const float s = S[a][b] * scale + bias_term(bias, h, i, j);
            if (pass == 0)
              acc = fmaxf(acc, s);
            else
              acc += expf(s - ref);
          }
        }
        if (pass == 0) {
          acc = group16_max(acc);
          if (tx == 0) row_m[r] = fmaxf(row_m[r], acc);
        } else if (pass == 1) {
          acc = group16_sum(acc);
          if (tx == 0) row_l[r] += acc;
        } else {
          part += acc;
        }
      }
      if (pass == 2) {
        part = warp_sum(part);
        if ((tid & 31) == 0) red[tid >> 5] = part;
        __syncthreads();
        if (tid == 0) {
          float t = 0.f;
          for (int w = 0; w < kThreads / 32; ++w) t += red[w];
          mass_s[J] = t / (float)BLK;
        }
      }
    }
    __syncthreads();
    if (pass == 1) {
      for (int r = tid; r < BLK; r += kThreads) {
        const float z = row_m[r] + logf(row_l[r]);
        row_m[r] = z;  // from here on row_m holds the log-normaliser
        const size_t gi = (size_t)h * L + (size_t)I * BLK + r;
        lse_ws[gi] = z;
        if (lse_out) lse_out[gi] = z;
      }
    }
    __syncthreads();
  }

  // ---- selection ----
  const int n = I + 1;
  if (tid < n) {
    const uint64_t kj = ((uint64_t)__float_as_uint(mass_s[tid]) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)tid);
    int rank = 0;
    for (int t = 0; t < n; ++t) {
      const uint64_t kt = ((uint64_t)__float_as_uint(mass_s[t]) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)t);
      rank += (kt > kj);
    }
    sorted_s[rank] = tid;
  }
  if (tid < 8) bits_s[tid] = 0u;
  __syncthreads();
  if (tid == 0) {
    double cum = 0.0;
    int k = 0;
    const double pd = (double)p;
    if (p >= 1.f) {
      for (k = 0; k < n; ++k) cum += (double)mass_s[sorted_s[k]];
    } else {
      while (k < n) {
        cum += (double)mass_s[sorted_s[k]];
        ++k;
        if (cum >= pd) break;
      }
    }
    kstar_s = k;
    kept_mass[u] = (float)cum;
    count_ws[u] = k;
  }
  __syncthreads();
  if (tid < kstar_s) atomicOr(&bits_s[sorted_s[tid] >> 5], 1u << (sorted_s[tid] & 31));
  __syncthreads();
  if (tid < nkw) kept_bits[(size_t)u * nkw + tid] = bits_s[tid];
  if (mass_out)
    for (int J = tid; J < nkb; J += kThreads) mass_out[(size_t)u * nkb + J] = (J <= I) ? mass_s[J] : 0.f;
  if (!renorm) return;
  // renormalised map: each row's kept mass, sum over kept blocks of exp(s - lse), is absorbed into
  // the normaliser the emit pass divides by
  for (int r = tid; r < BLK; r += kThreads) row_l[r] = 0.f;
  for (int J = 0; J <= I; ++J) {
    if (!((bits_s[J >> 5] >> (J & 31)) & 1u)) continue;
    __syncthreads();
    load_rows<T, BLK, D>(Ks, K + ((size_t)h * L + (size_t)J * BLK) * D, BLK);
    __syncthreads();
    float S[R][R];
    tile_dot<BLK, BLK, D>(Qs, Ks, S);
#pragma unroll
    for (int a = 0; a < R; ++a) {
      const int r = ty + 16 * a;
      const int i = I * BLK + r;
      float acc = 0.f;
#pragma unroll
      for (int b = 0; b < R; ++b) {
        const int j = J * BLK + tx + 16 * b;
        if (j <= i) acc += expf(S[a][b] * scale + bias_term(bias, h, i, j) - row_m[r]);
      }
      acc = group16_sum(acc);
      if (tx == 0) row_l[r] += acc;
    }
  }
  __syncthreads();
  for (int r = tid; r < BLK; r += kThreads)
    if (row_l[r] > 0.f) lse_ws[(size_t)h * L + (size_t)I * BLK + r] += logf(row_l[r]);
}

// ---------------------------------------------------------------------------------------------
// Compression, part 3: emit the kept tiles' probabilities P_ij = exp(s_ij - lse_i) (0 above the
// causal diagonal) at their BSR positions, and their column indices.
// ---------------------------------------------------------------------------------------------
template <typename T, typename TV, int BLK, int D>
__global__ void __launch_bounds__(kThreads) k_emit(
    const T* __restrict__ Q, const T* __restrict__ K, int H, int L, float scale, Bias bias,
    const float* __restrict__ lse_ws, const int32_t* __restrict__ row_ptr,
    const uint32_t* __restrict__ kept_bits, int64_t capacity, int32_t* __restrict__ col_idx,
    TV* __restrict__ vals, int qb_hi) {
  extern __shared__ float smem[];
  float* Qs = smem;
  float* Ks = Qs + BLK * (D + 1);
  __shared__ float lse_s[BLK];
  const int nqb = L / BLK, nkw = (nqb + 31) / 32;
  const int I = qb_hi - 1 - (int)(blockIdx.x / H);  // query blocks qb_hi - 1, qb_hi - 2, ...
  const int h = (int)(blockIdx.x % H);
  const int u = h * nqb + I;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  constexpr int R = BLK / 16;
  load_rows<T, BLK, D>(Qs, Q + ((size_t)h * L + (size_t)I * BLK) * D, BLK);
  for (int r = tid; r < BLK; r += kThreads) lse_s[r] = lse_ws[(size_t)h * L + (size_t)I * BLK + r];
  const uint32_t* bits = kept_bits + (size_t)u * nkw;
  int64_t t = row_ptr[u];
  for (int J = 0; J <= I; ++J) {
    if (!((bits[J >> 5] >> (J & 31)) & 1u)) continue;
    if (t < capacity) {
      __syncthreads();
      load_rows<T, BLK, D>(Ks, K + ((size_t)h * L + (size_t)J * BLK) * D, BLK);
      __syncthreads();
      float S[R][R];
      tile_dot<BLK, BLK, D>(Qs, Ks, S);
      TV* out = vals + (size_t)t * BLK * BLK;
#pragma unroll
      for (int a = 0; a < R; ++a) {
        const int r = ty + 16 * a;
        const int i = I * BLK + r;
#pragma unroll
        for (int b = 0; b < R; ++b) {
          const int c = tx + 16 * b;
          const int j = J * BLK + c;
          const float pr = (j <= i) ? expf(S[a][b] * scale + bias_term(bias, h, i, j) - lse_s[r]) : 0.f;
          out[tile_offset<TV>(r, c, BLK)] = from_f32<TV>(pr);
        }
      }
      if (tid == 0) col_idx[t] = J;
    }
    ++t;
  }
}

// Stored map values: element at storage offset `off` of tile t, as fp32, with its tile coordinates.
template <typename TM>
struct MapVals {
  const TM* vals;
  const float* scale;  // fp8 only
  __device__ __forceinline__ float at(int64_t t, int off, int B) const { return to_f32(vals[t * B * B + off]); }
  __device__ __forceinline__ void coords(int off, int B, int& a, int& b) const { tile_coords<TM>(off, B, a, b); }
};
template <>
struct MapVals<uint8_t> {
  const uint8_t* vals;
  const float* scale;
  __device__ __forceinline__ void coords(int off, int B, int& a, int& b) const {
    const int panel = off / (B * 64), rem = off - panel * B * 64;
    a = rem >> 6;
    b = panel * 64 + ((rem & 63) & ~3) + fp8_perm4(rem & 3);  // the order (0, 2, 1, 3) is its own inverse
  }
  __device__ __forceinline__ float at(int64_t t, int off, int B) const {
    int a, b;
    coords(off, B, a, b);
    const __half_raw h = __nv_cvt_fp8_to_halfraw(vals[t * B * B + off], __NV_E4M3);
    return __half2float(*reinterpret_cast<const __half*>(&h)) * scale[t * fp8_scales_per_tile(B) + fp8_scale_index(a, b, B)];
  }
};

// ---------------------------------------------------------------------------------------------
// Retrieval: O_r[I] = sum_{J <= I} X[I,J] V_r[J],  X = sum_s W[r,s] A_s[I,J] over kept tiles.
// One CTA per (query block, receiver head, request).  X is built in shared memory only.
// ---------------------------------------------------------------------------------------------
template <typename T, typename TM, int BLK, int DV>
__global__ void __launch_bounds__(kThreads) k_retrieve(
    const int32_t* __restrict__ row_ptr, const uint32_t* __restrict__ kept_bits,
    MapVals<TM> mv, int64_t capacity, int H_s, int L, const float* __restrict__ W,
    int H_r, const T* __restrict__ V, int64_t v_elems, T* __restrict__ O,
    const int64_t* __restrict__ v_req_off, int64_t v_req_stride, int64_t v_head_stride, int v_group,
    int qb_hi, const int32_t* __restrict__ v_pages, int page_rows, int pages_per_req, WsHeader* ws) {
  extern __shared__ float smem[];
  float* Xs = smem;                   // [BLK][BLK + 1]
  float* Vs = Xs + BLK * (BLK + 1);   // [BLK][DV + 1]
  __shared__ float Ws[64];
  const int nqb = L / BLK, nkw = (nqb + 31) / 32;
  const int I = qb_hi - 1 - (int)(blockIdx.x / H_r);
  const int r = (int)(blockIdx.x % H_r);
  const int q = blockIdx.y;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  constexpr int R = BLK / 16, C = DV / 16, E = BLK * BLK / kThreads;
  for (int s = tid; s < H_s; s += kThreads) Ws[s] = W[(size_t)r * H_s + s];
  // value head g = r / v_group of request q; rows 0 .. (I + 1) * BLK - 1 must lie inside the
  // allocation, else the request reads zeros and the status word records the bad offset
  const int g = r / v_group, H_v = H_r / v_group;
  const int64_t voff = v_pages ? 0 : (v_req_off ? v_req_off[q] : (int64_t)q * v_req_stride) + (int64_t)g * v_head_stride;
  bool v_ok = true;
  if (v_pages) {
    for (int pg = 0; pg <= ((I + 1) * BLK - 1) / page_rows; ++pg) {
      const int64_t page = v_pages[(int64_t)q * pages_per_req + pg];
      v_ok = v_ok && page >= 0 && (page * H_v + g + 1) * page_rows * DV <= v_elems;
    }
  } else {
    v_ok = voff >= 0 && voff + (int64_t)(I + 1) * BLK * DV <= v_elems;
  }
  if (!v_ok && tid == 0) set_status(ws, MR_ERR_DEVICE_CHECK, 4u);
  const T* Vr = V + (v_ok ? voff : 0);
  // element offset of value row j (paged: row j % page_rows of the request's page j / page_rows)
  auto vrow = [&](int j) -> const T* {
    if (!v_pages) return Vr + (int64_t)j * DV;
    const int64_t page = v_pages[(int64_t)q * pages_per_req + j / page_rows];
    return V + ((page * H_v + g) * page_rows + j % page_rows) * DV;
  };
  float acc[R][C];
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int c = 0; c < C; ++c) acc[a][c] = 0.f;
  __syncthreads();
  for (int J = 0; J <= (v_ok ? I : -1); ++J) {
    float x[E];
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = 0.f;
    bool any = false;
    for (int s = 0; s < H_s; ++s) {
      const int us = s * nqb + I;
      const uint32_t* bits = kept_bits + (size_t)us * nkw;
      if (!((bits[J >> 5] >> (J & 31)) & 1u)) continue;
      const int64_t t = (int64_t)row_ptr[us] + kept_rank(bits, J);
      if (t >= capacity) {  // the map overflowed: this tile was never stored
        if (tid == 0) set_status(ws, MR_ERR_CAPACITY, 2u);
        continue;
      }
      any = true;
      const float w = Ws[s];
#pragma unroll
      for (int e = 0; e < E; ++e) x[e] = fmaf(w, mv.at(t, tid + e * kThreads, BLK), x[e]);
    }
    if (!any) continue;
    __syncthreads();
#pragma unroll
    for (int e = 0; e < E; ++e) {
      int ra, cb;
      mv.coords(tid + e * kThreads, BLK, ra, cb);
      Xs[ra * (BLK + 1) + cb] = x[e];
    }
    for (int e = tid; e < BLK * DV; e += kThreads) {
      const int rr = e / DV, c = e - (e / DV) * DV;
      Vs[rr * (DV + 1) + c] = to_f32(vrow(J * BLK + rr)[c]);
    }
    __syncthreads();
#pragma unroll 4
    for (int j = 0; j < BLK; ++j) {
      float xv[R], vv[C];
#pragma unroll
      for (int a = 0; a < R; ++a) xv[a] = Xs[(ty + 16 * a) * (BLK + 1) + j];
#pragma unroll
      for (int c = 0; c < C; ++c) vv[c] = Vs[j * (DV + 1) + tx + 16 * c];
#pragma unroll
      for (int a = 0; a < R; ++a)
#pragma unroll
        for (int c = 0; c < C; ++c) acc[a][c] = fmaf(xv[a], vv[c], acc[a][c]);
    }
  }
  T* Or = O + ((size_t)q * H_r + r) * (size_t)L * DV;
#pragma unroll
  for (int a = 0; a < R; ++a)
#pragma unroll
    for (int c = 0; c < C; ++c)
      Or[(size_t)(I * BLK + ty + 16 * a) * DV + tx + 16 * c] = from_f32<T>(acc[a][c]);
}

// ---------------------------------------------------------------------------------------------
// Dense causal attention (online softmax), packed variable-length sequences.
// ---------------------------------------------------------------------------------------------
template <typename T, int D, int DV>
__global__ void __launch_bounds__(kThreads) k_dense(
    const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V, T* __restrict__ O,
    int total_q, int total_k, const int32_t* __restrict__ cu_q, const int32_t* __restrict__ cu_k,
    const int32_t* __restrict__ q_offset, int n_seq, float scale, Bias bias) {
  constexpr int BM = 64, BN = 64, RA = BM / 16, RB = BN / 16, C = DV / 16;
  extern __shared__ float smem[];
  float* Qs = smem;                 // [BM][D + 1]
  float* Ks = Qs + BM * (D + 1);    // [BN][D + 1]
  float* Vs = Ks + BN * (D + 1);    // [BN][DV + 1]
  float* Ps = Vs + BN * (DV + 1);   // [BM][BN + 1]
  const int h = blockIdx.y;
  int seq = -1, tin = 0;
  {
    int accum = 0;
    for (int s = 0; s < n_seq; ++s) {
      const int nt = (cu_q[s + 1] - cu_q[s] + BM - 1) / BM;
      if ((int)blockIdx.x < accum + nt) {
        seq = s;
        tin = blockIdx.x - accum;
        break;
      }
      accum += nt;
    }
  }
  if (seq < 0) return;
  const int q0 = cu_q[seq] + tin * BM;
  const int nq = min(BM, cu_q[seq + 1] - q0);
  const int k0 = cu_k[seq];
  const int nk = cu_k[seq + 1] - k0;
  const int off = q_offset ? q_offset[seq] : 0;
  const int pos0 = off + tin * BM;  // absolute position of the tile's first row
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  load_rows<T, BM, D>(Qs, Q + ((size_t)h * total_q + q0) * D, nq);
  float m[RA], l[RA], o[RA][C];
#pragma unroll
  for (int a = 0; a < RA; ++a) {
    m[a] = -INFINITY;
    l[a] = 0.f;
#pragma unroll
    for (int c = 0; c < C; ++c) o[a][c] = 0.f;
  }
  const int last = min(pos0 + nq - 1, nk - 1);
  const int n_kt = (last >= 0) ? last / BN + 1 : 0;
  for (int kt = 0; kt < n_kt; ++kt) {
    __syncthreads();
    const int krows = min(BN, nk - kt * BN);
    load_rows<T, BN, D>(Ks, K + ((size_t)h * total_k + k0 + (size_t)kt * BN) * D, krows);
    load_rows<T, BN, DV>(Vs, V + ((size_t)h * total_k + k0 + (size_t)kt * BN) * DV, krows);
    __syncthreads();
    float S[RA][RB];
    tile_dot<BM, BN, D>(Qs, Ks, S);
#pragma unroll
    for (int a = 0; a < RA; ++a) {
      const int rr = ty + 16 * a;
      const int pos = pos0 + rr;
      const bool valid = rr < nq;
      float sv[RB];
      float rmax = -INFINITY;
#pragma unroll
      for (int b = 0; b < RB; ++b) {
        const int j = kt * BN + tx + 16 * b;
        sv[b] = (valid && j <= pos && j < nk) ? S[a][b] * scale + bias_term(bias, h, pos, j) : -INFINITY;
        rmax = fmaxf(rmax, sv[b]);
      }
      rmax = group16_max(rmax);
      const float mn = fmaxf(m[a], rmax);
      const float corr = (mn == -INFINITY) ? 1.f : expf(m[a] - mn);
      float rs = 0.f;
#pragma unroll
      for (int b = 0; b < RB; ++b) {
        const float pv = (mn == -INFINITY) ? 0.f : expf(sv[b] - mn);
        Ps[rr * (BN + 1) + tx + 16 * b] = pv;
        rs += pv;
      }
      rs = group16_sum(rs);
      l[a] = l[a] * corr + rs;
      m[a] = mn;
#pragma unroll
      for (int c = 0; c < C; ++c) o[a][c] *= corr;
    }
    __syncthreads();
#pragma unroll 4
    for (int j = 0; j < BN; ++j) {
      float pv[RA], vv[C];
#pragma unroll
      for (int a = 0; a < RA; ++a) pv[a] = Ps[(ty + 16 * a) * (BN + 1) + j];
#pragma unroll
      for (int c = 0; c < C; ++c) vv[c] = Vs[j * (DV + 1) + tx + 16 * c];
#pragma unroll
      for (int a = 0; a < RA; ++a)
#pragma unroll
        for (int c = 0; c < C; ++c) o[a][c] = fmaf(pv[a], vv[c], o[a][c]);
    }
  }
#pragma unroll
  for (int a = 0; a < RA; ++a) {
    const int rr = ty + 16 * a;
    if (rr < nq) {
      const float inv = 1.f / l[a];
#pragma unroll
      for (int c = 0; c < C; ++c)
        O[((size_t)h * total_q + q0 + rr) * DV + tx + 16 * c] = from_f32<T>(o[a][c] * inv);
    }
  }
}

__global__ void k_scan_counts(const int* __restrict__ count, int n, int32_t* __restrict__ row_ptr,
                              int64_t* __restrict__ nnz, int64_t capacity, WsHeader* ws) {
  __shared__ long long warp_tot[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int beg = min(n, tid * per), end = min(n, beg + per);
  long long local = 0;
  for (int i = beg; i < end; ++i) local += count[i];
  long long incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x / 32;
    long long v = (lane < nw) ? warp_tot[lane] : 0;
    long long inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long t = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += t;
    }
    if (lane < nw) warp_tot[lane] = inc - v;  // exclusive
  }
  __syncthreads();
  long long base = warp_tot[warp] + incl - local;
  for (int i = beg; i < end; ++i) {
    row_ptr[i] = (int32_t)base;
    base += count[i];
  }
  if (tid == blockDim.x - 1) {
    row_ptr[n] = (int32_t)base;
    *nnz = base;
    if (base > capacity) set_status(ws, MR_ERR_CAPACITY, 1u);
  }
}

template <typename TV>
__global__ void k_export(const TV* __restrict__ vals, int64_t n_elems, int B, float* __restrict__ out) {
  const int64_t tsz = (int64_t)B * B;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n_elems; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = e / tsz;
    const int w = (int)(e - t * tsz);
    out[e] = to_f32(vals[t * tsz + tile_offset<TV>(w / B, w % B, B)]);
  }
}

// fp8 tiles: e4m3 value times the scale of its 32-row x 64-key piece
__global__ void k_export_fp8(const uint8_t* __restrict__ vals, const float* __restrict__ scale, int64_t n_elems,
                             int B, float* __restrict__ out) {
  const int64_t tsz = (int64_t)B * B;
  const MapVals<uint8_t> mv{vals, scale};
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n_elems; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = e / tsz;
    const int w = (int)(e - t * tsz);
    out[e] = mv.at(t, tile_offset_fp8(w / B, w % B, B), B);
  }
}

template <typename KernelT>
cudaError_t set_smem(KernelT k, size_t bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <typename T, typename TV, int BLK, int D>
cudaError_t compress_impl(const CompressArgs& a) {
  const int nqb = a.L / BLK;
  const size_t smem = (size_t)2 * BLK * (D + 1) * sizeof(float);
  auto k1 = k_compress_stats<T, BLK, D>;
  cudaError_t e = set_smem(k1, smem);
  if (e != cudaSuccess) return e;
  {
    ProfScope ps(kKCompressStats, a.stream);
    k1<<<a.H * (a.qb1 - a.qb0), kThreads, smem, a.stream>>>(
        (const T*)a.Q, (const T*)a.K, a.H, a.L, a.scale, a.p, a.bias, a.lse_ws, a.count_ws,
        a.map.kept_bits, a.map.kept_mass, a.map.mass, a.map.lse, a.qb1, a.map.renormalised);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = launch_scan_counts(a.count_ws, a.H * nqb, a.map, a.ws, a.stream)) != cudaSuccess) return e;
  auto k3 = k_emit<T, TV, BLK, D>;
  if ((e = set_smem(k3, smem)) != cudaSuccess) return e;
  {
    ProfScope ps(kKEmit, a.stream);
    k3<<<a.H * (a.qb1 - a.qb0), kThreads, smem, a.stream>>>(
        (const T*)a.Q, (const T*)a.K, a.H, a.L, a.scale, a.bias, a.lse_ws, a.map.row_ptr,
        a.map.kept_bits, a.map.capacity_tiles, a.map.col_idx, (TV*)a.map.vals, a.qb1);
  }
  return cudaGetLastError();
}

template <typename T, typename TV, int BLK, int D>
cudaError_t emit_impl(const CompressArgs& a) {
  const size_t smem = (size_t)2 * BLK * (D + 1) * sizeof(float);
  auto k3 = k_emit<T, TV, BLK, D>;
  cudaError_t e = set_smem(k3, smem);
  if (e != cudaSuccess) return e;
  ProfScope ps(kKEmit, a.stream);
  k3<<<a.H * (a.qb1 - a.qb0), kThreads, smem, a.stream>>>(
      (const T*)a.Q, (const T*)a.K, a.H, a.L, a.scale, a.bias, a.lse_ws, a.map.row_ptr,
      a.map.kept_bits, a.map.capacity_tiles, a.map.col_idx, (TV*)a.map.vals, a.qb1);
  return cudaGetLastError();
}

template <typename T, typename TM, int BLK, int DV>
cudaError_t retrieve_impl(const RetrieveArgs& a) {
  const size_t smem = (size_t)(BLK * (BLK + 1) + BLK * (DV + 1)) * sizeof(float);
  auto k = k_retrieve<T, TM, BLK, DV>;
  const MapVals<TM> mv{(const TM*)a.map.vals, a.map.tile_scale};
  cudaError_t e = set_smem(k, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.qb1 - a.qb0) * a.H_r, a.n_req);
  ProfScope ps(kKRetrieve, a.stream);
  k<<<grid, kThreads, smem, a.stream>>>(a.map.row_ptr, a.map.kept_bits, mv, a.map.capacity_tiles, a.map.H_s, a.map.L, a.W, a.H_r,
                                         (const T*)a.V, a.v_elems, (T*)a.O, a.v_req_off, a.v_req_stride,
                                         a.v_head_stride, a.v_group, a.qb1, a.v_pages, a.page_rows,
                                         a.pages_per_req, a.ws);
  return cudaGetLastError();
}

template <typename T, int D, int DV>
cudaError_t dense_impl(const DenseArgs& a, int total_k) {
  const size_t smem = (size_t)(64 * (D + 1) * 2 + 64 * (DV + 1) + 64 * 65) * sizeof(float);
  auto k = k_dense<T, D, DV>;
  cudaError_t e = set_smem(k, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.total_q / 64 + a.n_seq, a.H);
  ProfScope ps(kKDense, a.stream);
  k<<<grid, kThreads, smem, a.stream>>>((const T*)a.Q, (const T*)a.K, (const T*)a.V, (T*)a.O,
                                         a.total_q, total_k, a.cu_q, a.cu_k, a.q_offset, a.n_seq,
                                         a.scale, a.bias);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scan_counts(const int* count, int n, mr_bsr map, WsHeader* ws, cudaStream_t st) {
  ProfScope ps(kKScanCounts, st);
  k_scan_counts<<<1, 1024, 0, st>>>(count, n, map.row_ptr, map.nnz, map.capacity_tiles, ws);
  return cudaGetLastError();
}

cudaError_t simt_compress(const CompressArgs& a) {
  const bool bf = a.dt == MR_BF16;
  if (a.block == 64 && a.d == 64) return bf ? compress_impl<__nv_bfloat16, __nv_bfloat16, 64, 64>(a) : compress_impl<float, float, 64, 64>(a);
  if (a.block == 64 && a.d == 128) return bf ? compress_impl<__nv_bfloat16, __nv_bfloat16, 64, 128>(a) : compress_impl<float, float, 64, 128>(a);
  if (a.block == 128 && a.d == 64) return bf ? compress_impl<__nv_bfloat16, __nv_bfloat16, 128, 64>(a) : compress_impl<float, float, 128, 64>(a);
  if (a.block == 128 && a.d == 128) return bf ? compress_impl<__nv_bfloat16, __nv_bfloat16, 128, 128>(a) : compress_impl<float, float, 128, 128>(a);
  return cudaErrorInvalidValue;
}

cudaError_t simt_emit(const CompressArgs& a) {
  const bool bf = a.dt == MR_BF16;
  if (a.block == 64 && a.d == 64) return bf ? emit_impl<__nv_bfloat16, __nv_bfloat16, 64, 64>(a) : emit_impl<float, float, 64, 64>(a);
  if (a.block == 64 && a.d == 128) return bf ? emit_impl<__nv_bfloat16, __nv_bfloat16, 64, 128>(a) : emit_impl<float, float, 64, 128>(a);
  if (a.block == 128 && a.d == 64) return bf ? emit_impl<__nv_bfloat16, __nv_bfloat16, 128, 64>(a) : emit_impl<float, float, 128, 64>(a);
  if (a.block == 128 && a.d == 128) return bf ? emit_impl<__nv_bfloat16, __nv_bfloat16, 128, 128>(a) : emit_impl<float, float, 128, 128>(a);
  return cudaErrorInvalidValue;
}

cudaError_t simt_retrieve(const RetrieveArgs& a) {
  const bool bf = a.dt == MR_BF16;
  const int B = a.map.block;
  if (a.map.val_dtype == MR_FP8_E4M3) {  // bf16 values, fp8 map
    if (B == 64 && a.d_v == 64) return retrieve_impl<__nv_bfloat16, uint8_t, 64, 64>(a);
    if (B == 64 && a.d_v == 128) return retrieve_impl<__nv_bfloat16, uint8_t, 64, 128>(a);
    if (B == 128 && a.d_v == 64) return retrieve_impl<__nv_bfloat16, uint8_t, 128, 64>(a);
    if (B == 128 && a.d_v == 128) return retrieve_impl<__nv_bfloat16, uint8_t, 128, 128>(a);
    return cudaErrorInvalidValue;
  }
  if (B == 64 && a.d_v == 64) return bf ? retrieve_impl<__nv_bfloat16, __nv_bfloat16, 64, 64>(a) : retrieve_impl<float, float, 64, 64>(a);
  if (B == 64 && a.d_v == 128) return bf ? retrieve_impl<__nv_bfloat16, __nv_bfloat16, 64, 128>(a) : retrieve_impl<float, float, 64, 128>(a);
  if (B == 128 && a.d_v == 64) return bf ? retrieve_impl<__nv_bfloat16, __nv_bfloat16, 128, 64>(a) : retrieve_impl<float, float, 128, 64>(a);
  if (B == 128 && a.d_v == 128) return bf ? retrieve_impl<__nv_bfloat16, __nv_bfloat16, 128, 128>(a) : retrieve_impl<float, float, 128, 128>(a);
  return cudaErrorInvalidValue;
}

cudaError_t simt_dense(const DenseArgs& a) {
  const bool bf = a.dt == MR_BF16;
  const int tk = a.total_k;
  if (a.d == 64 && a.d_v == 64) return bf ? dense_impl<__nv_bfloat16, 64, 64>(a, tk) : dense_impl<float, 64, 64>(a, tk);
  if (a.d == 128 && a.d_v == 128) return bf ? dense_impl<__nv_bfloat16, 128, 128>(a, tk) : dense_impl<float, 128, 128>(a, tk);
  if (a.d == 64 && a.d_v == 128) return bf ? dense_impl<__nv_bfloat16, 64, 128>(a, tk) : dense_impl<float, 64, 128>(a, tk);
  if (a.d == 128 && a.d_v == 64) return bf ? dense_impl<__nv_bfloat16, 128, 64>(a, tk) : dense_impl<float, 128, 64>(a, tk);
  return cudaErrorInvalidValue;
}

cudaError_t launch_export(const mr_bsr& map, int64_t n_tiles, float* out, cudaStream_t st) {
  const int64_t n = n_tiles * (int64_t)map.block * map.block;
  if (n == 0) return cudaSuccess;
  const int blocks = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  ProfScope ps(kKExport, st);
  if (map.val_dtype == MR_FP8_E4M3)
    k_export_fp8<<<blocks, 256, 0, st>>>((const uint8_t*)map.vals, map.tile_scale, n, map.block, out);
  else if (map.val_dtype == MR_BF16)
    k_export<__nv_bfloat16><<<blocks, 256, 0, st>>>((const __nv_bfloat16*)map.vals, n, map.block, out);
  else
    k_export<float><<<blocks, 256, 0, st>>>((const float*)map.vals, n, map.block, out);
  return cudaGetLastError();
}

}  // namespace mr
