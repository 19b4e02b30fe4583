// C-ABI of libmr: argument validation, workspace layout, status handling and kernel selection.
// Every check here runs on the host before anything is enqueued.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>

#include "../../include/mr.h"
#include "common.cuh"
#include "kernels.h"

using namespace mr;

namespace mr {
void debug_waits(uint64_t* wait_ns, int* skip_arrive);
}

namespace {

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct CompressLayout {
  size_t lse_off, count_off, total;
};

CompressLayout compress_layout(int H, int L, int block) {
  CompressLayout c;
  const size_t nqb = (size_t)(L / block);
  c.lse_off = kWsHeaderBytes;
  c.count_off = c.lse_off + align256((size_t)H * L * sizeof(float));
  c.total = c.count_off + align256((size_t)H * nqb * sizeof(int));
  return c;
}

bool shape_ok(int H, int L, int d, int block) {
  if (H < 1 || H > 64 || L < 1) return false;
  if (block != 64 && block != 128) return false;
  if (d != 64 && d != 128) return false;
  if (L % block != 0 || L / block > 256) return false;
  return true;
}

mr_status bias_ok(const mr_logit_bias* b, int keys) {
  if (!b) return MR_OK;
  if (b->sink_len < 0 || b->window < 0) return MR_ERR_INVALID_ARG;
  if (!isfinite(b->sink_bias) || !isfinite(b->window_bias)) return MR_ERR_INVALID_ARG;
  if (b->kb_bias) {
    if (b->kb_block <= 0) return MR_ERR_INVALID_ARG;
    if ((int64_t)b->n_kb * b->kb_block < keys) return MR_ERR_INVALID_ARG;
  }
  return MR_OK;
}

mr_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MR_OK : MR_ERR_CUDA; }

std::atomic<uint64_t> g_debug_wait_ns{0};
std::atomic<int> g_debug_skip{0};

// Clear the workspace header (status word and work-queue counters) in stream order.
cudaError_t reset_header(void* ws, cudaStream_t st) { return cudaMemsetAsync(ws, 0, sizeof(WsHeader), st); }

}  // namespace

void mr::debug_waits(uint64_t* wait_ns, int* skip_arrive) {
  *wait_ns = g_debug_wait_ns.load();
  *skip_arrive = g_debug_skip.load();
}

extern "C" {

int mr_version(void) { return 100; }

const char* mr_status_string(mr_status s) {
  switch (s) {
    case MR_OK: return "ok";
    case MR_ERR_INVALID_ARG: return "invalid argument";
    case MR_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case MR_ERR_CAPACITY: return "map capacity exceeded";
    case MR_ERR_CUDA: return "CUDA error";
    case MR_ERR_TIMEOUT: return "device wait timed out";
    case MR_ERR_DEVICE_CHECK: return "device check failed";
    case MR_ERR_RANGE: return "logit range too wide";
  }
  return "unknown status";
}

int mr_checked_build(void) { return mr::kCheckedBuild ? 1 : 0; }

int mr_device_supported(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return 0;
  return (major == 10 && minor == 0) ? 1 : 0;
}

size_t mr_compress_workspace_bytes(int H_s, int L, int d, int block) {
  if (!shape_ok(H_s, L, d, block)) return 0;
  return compress_layout(H_s, L, block).total;
}

int64_t mr_bsr_max_tiles(int H_s, int L, int block) {
  if (H_s < 1 || L < 1 || block < 1 || L % block) return 0;
  const int64_t nqb = L / block;
  return (int64_t)H_s * nqb * (nqb + 1) / 2;
}

mr_status mr_compress_blocks(const void* Q, const void* K, mr_dtype dt, int H_s, int L, int d,
                             float scale, float p, const mr_logit_bias* bias, int qb_begin,
                             int qb_end, mr_bsr* out, void* ws, size_t ws_bytes, void* stream) {
  if (!Q || !K || !out || !ws) return MR_ERR_INVALID_ARG;
  if (dt != MR_BF16 && dt != MR_F32) return MR_ERR_INVALID_ARG;
  if (!isfinite(scale) || !(p > 0.f) || isnan(p)) return MR_ERR_INVALID_ARG;
  if (H_s < 1 || L < 1) return MR_ERR_INVALID_ARG;
  if (out->block < 1 || L % out->block) return MR_ERR_UNSUPPORTED;
  if (!shape_ok(H_s, L, d, out->block)) return MR_ERR_UNSUPPORTED;
  if (out->H_s != H_s || out->L != L) return MR_ERR_INVALID_ARG;
  const bool fp8 = out->val_dtype == MR_FP8_E4M3;
  if (out->val_dtype != dt && !(fp8 && dt == MR_BF16)) return MR_ERR_UNSUPPORTED;
  if (fp8 && d != 128) return MR_ERR_UNSUPPORTED;  // fp8 maps come from the tensor-core emit only
  if (fp8 && out->capacity_tiles > 0 && !out->tile_scale) return MR_ERR_INVALID_ARG;
  if (out->capacity_tiles < 0) return MR_ERR_INVALID_ARG;
  if (!out->row_ptr || !out->kept_mass || !out->kept_bits || !out->nnz) return MR_ERR_INVALID_ARG;
  if (out->capacity_tiles > 0 && (!out->col_idx || !out->vals)) return MR_ERR_INVALID_ARG;
  if (mr_bsr_max_tiles(H_s, L, out->block) >= ((int64_t)1 << 31)) return MR_ERR_UNSUPPORTED;
  const int nqb = L / out->block;
  if (qb_begin < 0 || qb_end > nqb || qb_begin >= qb_end) return MR_ERR_INVALID_ARG;
  const mr_status bs = bias_ok(bias, L);
  if (bs != MR_OK) return bs;
  const CompressLayout lay = compress_layout(H_s, L, out->block);
  if (ws_bytes < lay.total) return MR_ERR_INVALID_ARG;

  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = reset_header(ws, st);
  if (e != cudaSuccess) return MR_ERR_CUDA;
  CompressArgs a;
  a.Q = Q;
  a.K = K;
  a.dt = dt;
  a.H = H_s;
  a.L = L;
  a.d = d;
  a.block = out->block;
  a.scale = scale;
  a.p = p;
  a.bias = make_bias(bias);
  a.ws = (WsHeader*)ws;
  a.lse_ws = (float*)((char*)ws + lay.lse_off);
  a.count_ws = (int*)((char*)ws + lay.count_off);
  a.qb0 = qb_begin;
  a.qb1 = qb_end;
  a.map = *out;
  a.stream = st;
  if (qb_begin > 0 || qb_end < nqb) {
    // rows outside the range are empty: zero counts, kept bits, kept masses (and stored masses)
    const size_t rows = (size_t)H_s * nqb, words = (size_t)(nqb + 31) / 32;
    if (cudaMemsetAsync(a.count_ws, 0, rows * sizeof(int), st) != cudaSuccess ||
        cudaMemsetAsync(out->kept_bits, 0, rows * words * sizeof(uint32_t), st) != cudaSuccess ||
        cudaMemsetAsync(out->kept_mass, 0, rows * sizeof(float), st) != cudaSuccess ||
        (out->mass && cudaMemsetAsync(out->mass, 0, rows * nqb * sizeof(float), st) != cudaSuccess))
      return MR_ERR_CUDA;
  }
  if (!tc_compress_supported(a)) return fp8 ? MR_ERR_UNSUPPORTED : from_cuda(simt_compress(a));
  if ((e = tc_compress_stats(a)) != cudaSuccess) return MR_ERR_CUDA;
  if ((e = launch_scan_counts(a.count_ws, H_s * nqb, a.map, a.ws, st)) != cudaSuccess) return MR_ERR_CUDA;
  return from_cuda(tc_emit(a));
}

mr_status mr_compress(const void* Q, const void* K, mr_dtype dt, int H_s, int L, int d, float scale,
                      float p, const mr_logit_bias* bias, mr_bsr* out, void* ws, size_t ws_bytes,
                      void* stream) {
  if (!out) return MR_ERR_INVALID_ARG;
  if (out->block < 1 || L < 1 || L % out->block) return L < 1 ? MR_ERR_INVALID_ARG : MR_ERR_UNSUPPORTED;
  return mr_compress_blocks(Q, K, dt, H_s, L, d, scale, p, bias, 0, L / out->block, out, ws, ws_bytes, stream);
}

size_t mr_retrieve_workspace_bytes(const mr_bsr* map, int H_r, int d_v, int n_req) {
  (void)map;
  (void)H_r;
  (void)d_v;
  (void)n_req;
  return kRetrieveWsBytes;
}

mr_status mr_retrieve(const mr_bsr* map, const float* W, int H_r, const void* V, int64_t v_elems,
                      void* O, mr_dtype dt, int d_v, int n_req, const int64_t* v_req_off,
                      int64_t v_req_stride, int64_t v_head_stride, const mr_retrieve_opts* opts,
                      void* ws, size_t ws_bytes, void* stream) {
  if (!map || !W || !V || !O || !ws) return MR_ERR_INVALID_ARG;
  if (dt != MR_BF16 && dt != MR_F32) return MR_ERR_INVALID_ARG;
  if (H_r < 1 || n_req < 1 || v_head_stride < 0 || v_req_stride < 0 || v_elems < 1) return MR_ERR_INVALID_ARG;
  if (H_r > 256) return MR_ERR_UNSUPPORTED;
  if (d_v != 64 && d_v != 128) return MR_ERR_UNSUPPORTED;
  if (!shape_ok(map->H_s, map->L, 64, map->block)) return MR_ERR_UNSUPPORTED;
  const bool fp8 = map->val_dtype == MR_FP8_E4M3;
  if (map->val_dtype != dt && !(fp8 && dt == MR_BF16)) return MR_ERR_UNSUPPORTED;
  if (!map->row_ptr || !map->kept_bits || !map->vals) return MR_ERR_INVALID_ARG;
  if (fp8 && !map->tile_scale) return MR_ERR_INVALID_ARG;
  const int nqb = map->L / map->block;
  int qb0 = 0, qb1 = nqb, group = 1;
  const int32_t* pages = nullptr;
  int page_rows = 0, pages_per_req = 0;
  if (opts && opts->v_pages) {
    pages = opts->v_pages;
    page_rows = opts->page_rows;
    pages_per_req = opts->pages_per_req;
    if (page_rows < 64 || page_rows % 64 || pages_per_req < 1 ||
        (int64_t)pages_per_req * page_rows < map->L)
      return MR_ERR_INVALID_ARG;
  }
  if (opts) {
    if (opts->qb_begin != 0 || opts->qb_end != 0) {
      qb0 = opts->qb_begin;
      qb1 = opts->qb_end;
      if (qb0 < 0 || qb1 > nqb || qb0 >= qb1) return MR_ERR_INVALID_ARG;
    }
    if (opts->v_group < 0) return MR_ERR_INVALID_ARG;
    group = opts->v_group > 1 ? opts->v_group : 1;
    if (H_r % group) return MR_ERR_INVALID_ARG;
  }
  const int H_v = H_r / group;
  const int64_t seq = (int64_t)map->L * d_v;
  if (!(opts && opts->v_pages) && H_v > 1 && v_head_stride < seq) return MR_ERR_INVALID_ARG;
  // strided values: the furthest element read must lie inside the allocation
  if (pages) {
    if ((int64_t)page_rows * d_v * H_v > v_elems) return MR_ERR_INVALID_ARG;  // not even one page fits
  } else if (!v_req_off) {
    const int64_t last = (int64_t)(n_req - 1) * v_req_stride + (int64_t)(H_v - 1) * v_head_stride + seq;
    if (last > v_elems) return MR_ERR_INVALID_ARG;
  } else if (seq > v_elems) {
    return MR_ERR_INVALID_ARG;
  }
  if (ws_bytes < mr_retrieve_workspace_bytes(map, H_r, d_v, n_req)) return MR_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemsetAsync(ws, 0, kRetrieveWsBytes, st) != cudaSuccess) return MR_ERR_CUDA;  // header + progress
  RetrieveArgs a;
  a.map = *map;
  a.W = W;
  a.H_r = H_r;
  a.V = V;
  a.v_elems = v_elems;
  a.O = O;
  a.dt = dt;
  a.d_v = d_v;
  a.n_req = n_req;
  a.v_req_off = v_req_off;
  a.v_req_stride = v_req_stride;
  a.v_head_stride = v_head_stride;
  a.v_group = group;
  a.qb0 = qb0;
  a.qb1 = qb1;
  a.v_pages = pages;
  a.page_rows = page_rows;
  a.pages_per_req = pages_per_req;
  a.ws = (WsHeader*)ws;
  a.stream = st;
  return from_cuda(tc_retrieve_supported(a) ? tc_retrieve(a) : simt_retrieve(a));
}

size_t mr_dense_ref_workspace_bytes(int n_seq) {
  (void)n_seq;
  return kWsHeaderBytes;
}

mr_status mr_dense_ref(const void* Q, const void* K, const void* V, void* O, mr_dtype dt, int H,
                       int d, int d_v, const int32_t* cu_q, const int32_t* cu_k,
                       const int32_t* q_offset, int n_seq, int total_q, int total_k, float scale,
                       const mr_logit_bias* bias, void* ws, size_t ws_bytes, void* stream) {
  if (!Q || !K || !V || !O || !cu_q || !cu_k || !ws) return MR_ERR_INVALID_ARG;
  if (dt != MR_BF16 && dt != MR_F32) return MR_ERR_INVALID_ARG;
  if (H < 1 || n_seq < 1 || total_q < 0 || total_k < 1 || !isfinite(scale)) return MR_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || (d_v != 64 && d_v != 128)) return MR_ERR_UNSUPPORTED;
  const mr_status bs = bias_ok(bias, total_k);
  if (bs != MR_OK) return bs;
  if (ws_bytes < mr_dense_ref_workspace_bytes(n_seq)) return MR_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (reset_header(ws, st) != cudaSuccess) return MR_ERR_CUDA;
  if (total_q == 0) return MR_OK;
  DenseArgs a;
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.O = O;
  a.dt = dt;
  a.H = H;
  a.d = d;
  a.d_v = d_v;
  a.cu_q = cu_q;
  a.cu_k = cu_k;
  a.q_offset = q_offset;
  a.n_seq = n_seq;
  a.total_q = total_q;
  a.total_k = total_k;
  a.scale = scale;
  a.bias = make_bias(bias);
  a.ws = (WsHeader*)ws;
  a.stream = st;
  return from_cuda(tc_dense_supported(a) ? tc_dense(a) : simt_dense(a));
}

mr_status mr_sync_status(void* ws, void* stream) {
  if (!ws) return MR_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MR_ERR_CUDA;
  uint32_t code = 0;
  if (cudaMemcpy(&code, ws, sizeof(code), cudaMemcpyDeviceToHost) != cudaSuccess) return MR_ERR_CUDA;
  return (mr_status)code;
}

mr_status mr_bsr_nnz(const mr_bsr* map, int64_t* nnz_host, void* stream) {
  if (!map || !map->nnz || !nnz_host) return MR_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyAsync(nnz_host, map->nnz, sizeof(int64_t), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MR_ERR_CUDA;
  return from_cuda(cudaStreamSynchronize(st));
}

mr_status mr_bsr_export(const mr_bsr* map, int64_t n_tiles, float* out, void* stream) {
  if (!map || !out || n_tiles < 0 || (n_tiles > 0 && !map->vals)) return MR_ERR_INVALID_ARG;
  if (map->val_dtype == MR_FP8_E4M3 && n_tiles > 0 && !map->tile_scale) return MR_ERR_INVALID_ARG;
  if (n_tiles > map->capacity_tiles) return MR_ERR_INVALID_ARG;
  return from_cuda(launch_export(*map, n_tiles, out, (cudaStream_t)stream));
}

mr_status mr_gather_probe(const mr_bsr* map, int readers, int ring_slots, void* ws, size_t ws_bytes,
                          void* stream) {
  if (!map || !ws || readers < 1 || readers > 1024 || ws_bytes < kWsHeaderBytes) return MR_ERR_INVALID_ARG;
  if (ring_slots < 2 || ring_slots > 24 || ring_slots % 2) return MR_ERR_INVALID_ARG;
  if (!shape_ok(map->H_s, map->L, 64, map->block)) return MR_ERR_UNSUPPORTED;
  if (!map->row_ptr || !map->kept_bits || !map->vals) return MR_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (reset_header(ws, st) != cudaSuccess) return MR_ERR_CUDA;
  return from_cuda(launch_gather_probe(*map, readers, ring_slots, (WsHeader*)ws, st));
}

mr_status mr_debug_set(uint64_t wait_ns, int skip_arrive) {
  if (skip_arrive < 0 || skip_arrive > 1) return MR_ERR_INVALID_ARG;
  g_debug_wait_ns.store(wait_ns);
  g_debug_skip.store(skip_arrive);
  return MR_OK;
}

}  // extern "C"
