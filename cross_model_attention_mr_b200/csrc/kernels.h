// Host-side launchers of the libmr kernels (internal to the library; not part of the C-ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace mr {

struct CompressArgs {
  const void* Q;
  const void* K;
  mr_dtype dt;
  int H, L, d, block;
  float scale, p;
  Bias bias;
  WsHeader* ws;
  float* lse_ws;    // [H][L] natural-log row normaliser (workspace)
  int* count_ws;    // [H * nqb]
  int qb0, qb1;     // query blocks processed: qb0 <= I < qb1
  mr_bsr map;
  cudaStream_t stream;
};

struct RetrieveArgs {
  mr_bsr map;
  const float* W;
  int H_r;
  const void* V;
  int64_t v_elems;  // elements of the V allocation: every value read stays below it
  void* O;
  mr_dtype dt;
  int d_v, n_req;
  const int64_t* v_req_off;
  int64_t v_req_stride, v_head_stride;
  int v_group;      // receiver heads per value head
  int qb0, qb1;     // output query blocks: qb0 <= I < qb1
  const int32_t* v_pages;  // paged values: [n_req][pages_per_req] page numbers, or nullptr
  int page_rows, pages_per_req;
  WsHeader* ws;
  cudaStream_t stream;
};

struct DenseArgs {
  const void* Q;
  const void* K;
  const void* V;
  void* O;
  mr_dtype dt;
  int H, d, d_v;
  const int32_t* cu_q;
  const int32_t* cu_k;
  const int32_t* q_offset;
  int n_seq, total_q, total_k;
  float scale;
  Bias bias;
  WsHeader* ws;
  cudaStream_t stream;
};

// SIMT (CUDA-core) kernels: fp32 inputs, and bf16 where no tensor-core kernel applies.
cudaError_t simt_compress(const CompressArgs& a);
cudaError_t simt_emit(const CompressArgs& a);  // emit pass only (after statistics and scan)
cudaError_t simt_retrieve(const RetrieveArgs& a);
cudaError_t simt_dense(const DenseArgs& a);

// Tensor-core kernels (bf16, sm_100a).
bool tc_compress_supported(const CompressArgs& a);
cudaError_t tc_compress_stats(const CompressArgs& a);  // row normalisers, masses, selection
cudaError_t tc_emit(const CompressArgs& a);            // kept tiles -> map storage
bool tc_retrieve_supported(const RetrieveArgs& a);
cudaError_t tc_retrieve(const RetrieveArgs& a);
bool tc_dense_supported(const DenseArgs& a);
cudaError_t tc_dense(const DenseArgs& a);

// Failure-path test hook (mr_debug_set): wait limit for the dense kernel's protocol waits (0 = the
// default 2 s) and whether its softmax withholds its first "P ready" arrive.
void debug_waits(uint64_t* wait_ns, int* skip_arrive);

// Shared by every compress path: exclusive scan of the kept counts into row_ptr, nnz, capacity.
cudaError_t launch_scan_counts(const int* count, int n, mr_bsr map, WsHeader* ws, cudaStream_t st);

cudaError_t launch_export(const mr_bsr& map, int64_t n_tiles, float* out, cudaStream_t st);

// Measurement: the retrieval's map reads alone (each kept tile moved to shared memory `readers` times).
cudaError_t launch_gather_probe(const mr_bsr& map, int readers, int ring_slots, WsHeader* ws, cudaStream_t st);

}  // namespace mr
