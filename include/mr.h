/*
 * libmr: block-level top-p compression of causal attention maps and fused translated retrieval
 * for cross-model attention-map reuse, on NVIDIA B200 (sm_100a).
 *
 * The method is MapFlow ("Accelerating Cross-Model LLM Inference via Attention Map Reuse"):
 *   - a sender's per-head causal softmax maps are compressed once, per (layer, head, query
 *     block), to the smallest set of key blocks whose probability mass reaches p, and stored in
 *     Block Sparse Row form (sections 4 and 5.2, "Attention State Compressor");
 *   - a receiver head's map is a non-negative, normalised linear mix of sender heads' maps
 *     (section 3.3) and is applied to the receiver's values by one fused kernel that never writes
 *     the translated map to global memory (section 5.4, "Attention Retrieval with Fused Kernel").
 * mr_dense_ref is exact causal attention, softmax(QK^T/sqrt(d))V ("AttnCache Guide", section
 * "The Quadratic Self-Attention Cost"), for rows that are not reused and as the p = 1 reference.
 *
 * Conventions for every entry point:
 *   - All tensors are caller-owned device memory unless a parameter says "host".  The library
 *     allocates no memory and frees nothing.
 *   - Arguments are validated on the host before any launch; a rejected call returns
 *     MR_ERR_INVALID_ARG or MR_ERR_UNSUPPORTED and launches nothing.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream) with no
 *     host synchronisation.  Conditions found on the device (capacity overflow, a bounded wait
 *     that ran out, a failed device check) are recorded in a status word inside the workspace;
 *     read it with mr_sync_status.
 *   - No exception crosses the ABI.  Device code never traps or asserts.
 *   - Layouts are head-major and row-contiguous: element (h, row, c) of a [H][rows][dim]
 *     tensor is at ((h * rows) + row) * dim + c.
 */
#ifndef MR_H_
#define MR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MR_OK = 0,
  MR_ERR_INVALID_ARG = 1,  /* null pointer, bad size or value (host check, nothing launched) */
  MR_ERR_UNSUPPORTED = 2,  /* well-formed but outside this build: dtype, head dim, block, length */
  MR_ERR_CAPACITY = 3,     /* the compressed map needs more tiles than capacity_tiles (device) */
  MR_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  MR_ERR_TIMEOUT = 5,      /* a bounded device-side wait ran out; the kernel returned early */
  MR_ERR_DEVICE_CHECK = 6, /* a device-side consistency check failed */
  MR_ERR_RANGE = 7         /* a row's logits span too wide a range for the fp32 exponent path */
} mr_status;

/*
 * Element types.  MR_FP8_E4M3 is a map value type only (inputs stay MR_BF16): MapFlow section 9,
 * "Compact representations for reusable attention state".  An fp8 map stores each value as e4m3
 * (IEEE-style, 4 exponent bits with bias 7, 3 mantissa bits) times a float scale per 32-row x 64-key
 * piece of a tile (mr_bsr.tile_scale).
 */
typedef enum { MR_BF16 = 0, MR_F32 = 1, MR_FP8_E4M3 = 2 } mr_dtype;

/*
 * Synthetic causal logit bias b(h, i, j), added to sigma * q_i.k_j for j <= i.  It stands in for
 * the attention-sink, local-window and retrieval-head patterns the AttnCache page describes
 * ("The Attention Map Redundancy Discovery").  b is the MAXIMUM of the terms that apply, 0 when
 * none applies:
 *   sink_bias    when j < sink_len                (sink_len = 0 disables it)
 *   window_bias  when i - j < window              (window = 0 disables it)
 *   kb_bias[h * n_kb + j / kb_block]  when that device float is finite (-inf = no bias).
 * For mr_dense_ref, i is the absolute position q_offset + row.  Pass NULL for "no bias".
 */
typedef struct {
  int32_t sink_len;
  float sink_bias;
  int32_t window;
  float window_bias;
  const float* kb_bias; /* device [n_heads][n_kb] or NULL */
  int32_t kb_block;     /* keys per kb_bias entry (> 0 when kb_bias != NULL) */
  int32_t n_kb;         /* entries per head row (>= ceil(keys / kb_block)) */
} mr_logit_bias;

/*
 * Block Sparse Row map of one layer's H_s sender heads (MapFlow section 4: "Block Sparse Row
 * format").  Rows are (head h, query block I), numbered u = h * nqb + I with nqb = L / block;
 * columns are key blocks J <= I, nkb = L / block, nkb_words = ceil(nkb / 32).
 * The caller fills H_s, L, block, val_dtype, capacity_tiles and the pointers; mr_compress fills
 * the arrays.
 *   row_ptr   int32  [H_s * nqb + 1]  exclusive prefix sum of kept counts (row_ptr[0] = 0)
 *   col_idx   int32  [capacity_tiles] kept key-block indices, ascending within each row
 *   vals      [capacity_tiles][block * block] probabilities in val_dtype; tile t belongs to
 *             the row u with row_ptr[u] <= t < row_ptr[u+1] and column col_idx[t]; element (a, b)
 *             of a tile is the probability of query I*block + a on key J*block + b; entries above
 *             the causal diagonal are 0.  Values are not renormalised.  Storage order inside a
 *             tile: panels of P = 128 / sizeof(element) columns, each panel holding its `block`
 *             rows of 128 bytes in turn; in row a, the 16-byte chunk c of the panel is stored at
 *             chunk position c ^ (a % 8).  So element (a, b) sits at
 *               (b / P) * block * P + a * P + E * (((b % P) / E) ^ (a % 8)) + b % E,
 *             E = 16 / sizeof(element).  (Each panel is a 128-byte-swizzled MMA operand.)
 *             MR_FP8_E4M3 tiles are stored in panels of 64 columns, each panel holding its `block`
 *             rows of 64 bytes in turn with no swizzle, and within every group of 4 columns the
 *             bytes ordered (0, 2, 1, 3): element (a, b) at
 *               (b / 64) * block * 64 + a * 64 + (b % 64) - (b % 4) + perm(b % 4), perm = {0, 2, 1, 3},
 *             and the value is e4m3(a, b) * tile_scale[t * S + (a / 32) * (block / 64) + b / 64],
 *             S = (block / 32) * (block / 64) scales per tile.
 *             mr_bsr_export converts tiles to plain row-major fp32.
 *   kept_mass float  [H_s * nqb]      mass of the kept blocks (fp64 sum, rounded to fp32)
 *   kept_bits uint32 [H_s * nqb][nkb_words]  bit (J % 32) of word J / 32 set iff block J kept
 *   mass      float  [H_s * nqb][nkb] optional block masses (NULL = not written); J > I is 0
 *   lse       float  [H_s][L]         optional natural-log row normaliser log(sum_j exp(s_ij))
 *   nnz       int64  [1]              number of kept tiles (may exceed capacity_tiles)
 *   tile_scale float [capacity_tiles][S]  MR_FP8_E4M3 maps only (else unused, may be NULL): the
 *             scale of each 32-row x 64-key piece, max(piece) / 448 (448 = largest e4m3 value)
 *   renormalised  set by the caller before mr_compress: 0 stores the kept probabilities as they
 *             are (each row of the map then sums to its kept mass, at most 1); 1 stores every row
 *             divided by its kept mass, so a head's kept probabilities of each query sum to 1 (the
 *             renormalised top-p map; the pages leave renormalisation open).  Masses, selection and
 *             lse are the same either way.
 */
typedef struct {
  int32_t H_s;
  int32_t L;
  int32_t block;
  mr_dtype val_dtype;
  int64_t capacity_tiles;
  int32_t* row_ptr;
  int32_t* col_idx;
  void* vals;
  float* kept_mass;
  uint32_t* kept_bits;
  float* mass;
  float* lse;
  int64_t* nnz;
  float* tile_scale;
  int32_t renormalised;
} mr_bsr;

/* Library version (major * 100 + minor). */
int mr_version(void);

/* Human-readable name of a status code (static string). */
const char* mr_status_string(mr_status s);

/* 1 when the current device is sm_100 (B200-class) and the kernels can run, else 0. */
int mr_device_supported(void);

/*
 * 1 in the bounds-checked build of the library (libmr_checked.so), else 0.  That build checks the
 * index of every global store of the tensor-core kernels, and of every map read whose index comes
 * from device data, against the extents passed in; a miss skips the access and records
 * MR_ERR_DEVICE_CHECK with a site code in the workspace status.  Same entry points and results.
 */
int mr_checked_build(void);

/*
 * Workspace bytes mr_compress needs for this shape (device memory, 256-byte aligned, contents
 * need no initialisation).  Returns 0 for an unsupported shape.
 */
size_t mr_compress_workspace_bytes(int H_s, int L, int d, int block);

/*
 * Worst-case tile count of a map of this shape: every causal tile kept,
 * H_s * nqb * (nqb + 1) / 2.  A capacity of this size can never overflow.
 */
int64_t mr_bsr_max_tiles(int H_s, int L, int block);

/*
 * Compress one layer: MapFlow sections 4 and 5.2.
 *   Q, K   [H_s][L][d] in dtype dt (MR_BF16: bf16; MR_F32: fp32)
 *   scale  logit scale sigma (pass 1/sqrt(d) for standard attention)
 *   p      top-p threshold in (0, 1]; p >= 1 keeps every causal block.  The kept set of row
 *          (h, I) is the first k blocks of J = 0..I ordered by block mass descending (ties: the
 *          smaller J first), k the least count whose cumulative mass (fp64) is >= p.
 *          Block mass M_IJ = (1/block) * sum over the block's B x B probabilities.
 *   bias   optional logit bias (NULL = none); kb_bias rows are per sender head.
 *   out    map descriptor (see mr_bsr); out->H_s, L, block must equal the arguments.
 *   ws     workspace of at least mr_compress_workspace_bytes(H_s, L, d, block) bytes.
 * Supported: d in {64, 128}; block in {64, 128}; L a positive multiple of block with
 * L / block <= 256; H_s <= 64.  MR_BF16 maps use bf16 vals; MR_F32 maps use fp32 vals; bf16 inputs
 * with d = 128 may also write an MR_FP8_E4M3 map (out->val_dtype = MR_FP8_E4M3, out->tile_scale
 * set), whose values carry the e4m3 rounding error (at most 2^-4 relative, plus 2^-10 of their
 * piece's scale below the normal range).
 * bf16 with d = 128 (and per-key-block biases, if any, on multiples of 32 keys) runs on the
 * tensor-core kernels; other shapes on the CUDA-core kernels.  Either way vals hold the tiles in
 * the 128-byte-panel layout described at mr_bsr.
 * If the map needs more than capacity_tiles tiles, the status word records MR_ERR_CAPACITY and
 * no tile at or beyond capacity_tiles is written (nnz still reports the full count).
 */
mr_status mr_compress(const void* Q, const void* K, mr_dtype dt, int H_s, int L, int d,
                      float scale, float p, const mr_logit_bias* bias, mr_bsr* out, void* ws,
                      size_t ws_bytes, void* stream);

/*
 * mr_compress restricted to the query blocks qb_begin <= I < qb_end of every head (all heads, all
 * key blocks J <= I): MapFlow section 6 ("Chunked Prefill"), and the per-rank share of one sequence
 * split across GPUs by query-block range.  Rows of *out outside the range are written as empty
 * (count 0, no kept bits, kept mass 0); their row_ptr entries repeat the running total, so the
 * map is a valid BSR map of the whole layer whose only non-empty rows are the range's.  Row
 * normalisers in out->lse are written for the range's rows (and, for block 64, possibly for the
 * other block of a 128-row pair).  Needs the same workspace as mr_compress.  Requires
 * 0 <= qb_begin < qb_end <= L / block; mr_compress is this call with the full range.
 */
mr_status mr_compress_blocks(const void* Q, const void* K, mr_dtype dt, int H_s, int L, int d,
                             float scale, float p, const mr_logit_bias* bias, int qb_begin,
                             int qb_end, mr_bsr* out, void* ws, size_t ws_bytes, void* stream);

/*
 * Allocation-free variant of mr_compress.  The paper has no counterpart: this is a deployment
 * convenience of this library.
 *
 * Who needs it: callers that cannot allocate device memory, and so cannot hand mr_compress a
 * workspace.  Examples are code running inside a framework whose memory pool already owns the
 * GPU's memory (a raw allocation there fails or fragments the pool), plug-ins held to a fixed,
 * pre-planned memory budget, and serving loops that must not call the allocator once running.
 *
 * It computes exactly what mr_compress computes, with the same arguments except the workspace.
 * The scratch comes from one fixed array compiled into the library, of
 * MR_COMPRESS_NOALLOC_SCRATCH_BYTES bytes.  Every GPU that loads the library holds that array
 * until the process exits.  The call allocates and frees nothing; the caller still owns Q, K and
 * every array of *out.
 *   - Limit: shapes with mr_compress_workspace_bytes(H_s, L, d, out->block) larger than the array
 *     are rejected with MR_ERR_UNSUPPORTED before any work is enqueued.  That allows
 *     H_s * L <= 1048576 rows and H_s * (L / block) <= 16384 query blocks, e.g. 32 heads of 32768
 *     tokens.
 *   - First call on a device: it looks up the array's device address with that device current.
 *     Make the first call on each device before any stream capture begins.
 *   - All calls share the one array, which keeps the last call's contents.  Each call clears the
 *     parts that must start at zero, in stream order.  Calls whose work can overlap on the GPU
 *     (other streams or other host threads without ordering between them) race on the array and
 *     corrupt each other's maps: order them.
 *   - There is no caller-visible workspace: read the status word of the most recent call with
 *     mr_compress_noalloc_status (capacity overflow, a bounded wait that ran out).
 *   - The array's device address is cached per device for the life of its CUDA context; after
 *     cudaDeviceReset the cached address is stale, so do not call this entry point again in a
 *     process that reset a device it used.
 */
#define MR_COMPRESS_NOALLOC_SCRATCH_BYTES (256 + 4194304 + 65536)
mr_status mr_compress_noalloc(const void* Q, const void* K, mr_dtype dt, int H_s, int L, int d,
                              float scale, float p, const mr_logit_bias* bias, mr_bsr* out,
                              void* stream);

/*
 * Synchronise `stream` and return the device-side status that the most recent
 * mr_compress_noalloc call on the current device recorded in the fixed scratch array (MR_OK if
 * nothing failed).  Calls on other streams without ordering to `stream` may overwrite it.
 */
mr_status mr_compress_noalloc_status(void* stream);

/*
 * Workspace bytes mr_retrieve needs (device memory, 256-byte aligned): the status header and one
 * progress counter per CTA, which the CTAs of a schedule group read to stay together (the ones
 * that read the same map tiles then find them in L2).  mr_retrieve zeroes it before its launch;
 * calls that overlap on the GPU need separate workspaces.
 */
size_t mr_retrieve_workspace_bytes(const mr_bsr* map, int H_r, int d_v, int n_req);

/*
 * Options of mr_retrieve (pass NULL for the defaults: every query block, one V head per receiver
 * head).
 *   qb_begin, qb_end  compute only the output rows of query blocks qb_begin <= I < qb_end
 *                     (MapFlow section 6, "Chunked Prefill"; also one rank's share of a sequence
 *                     split across GPUs).  Output rows outside the range are not written.  Both 0:
 *                     every query block.  Otherwise 0 <= qb_begin < qb_end <= L / block.
 *   v_group           receiver heads that share one value head (grouped-query attention): receiver
 *                     head r reads value head r / v_group.  0 or 1: one value head per receiver
 *                     head.  H_r must be a multiple of v_group.
 *   v_pages           paged values (MapFlow section 6, "PagedAttention"), or NULL: device int32
 *                     [n_req][pages_per_req] page numbers.  Token j of request q is row
 *                     j % page_rows of page v_pages[q * pages_per_req + j / page_rows], and V is a
 *                     pool of pages laid out [page][H_v][page_rows][d_v] (H_v = H_r / v_group), so
 *                     element (q, g, j, c) is at
 *                     V + ((page * H_v + g) * page_rows + j % page_rows) * d_v + c.
 *                     v_req_off, v_req_stride and v_head_stride are then ignored.  page_rows: a
 *                     positive multiple of 64; pages_per_req * page_rows >= L.  A page number whose
 *                     rows fall outside [0, v_elems) reads zeros and records MR_ERR_DEVICE_CHECK.
 */
typedef struct {
  int32_t qb_begin;
  int32_t qb_end;
  int32_t v_group;
  const int32_t* v_pages;
  int32_t page_rows;
  int32_t pages_per_req;
} mr_retrieve_opts;

/*
 * Fused translated retrieval: MapFlow sections 3.3 and 5.4.
 *   O_r[i] = sum_{j <= i} ( sum_s W[r][s] * A_s[i][j] * [key block of j kept for (s, block of i)] )
 *            * V_g(r)[j],   g(r) = r / v_group
 * for every receiver head r < H_r, query row i < map->L (or of the options' query-block range) and
 * request q < n_req.  The translated map is formed tile by tile on chip and never written to
 * global memory.
 *   map     a map filled by mr_compress (its vals dtype equals dt, or is MR_FP8_E4M3 with dt = MR_BF16;
 *           fp8 maps are mixed in half precision from their e4m3 values)
 *   W       device fp32 [H_r][H_s], row r = receiver head r's weights over sender heads
 *   V       values in dtype dt: element (q, g, j, c) of value head g at
 *           V + v_off(q) + g * v_head_stride + j * d_v + c,
 *           v_off(q) = v_req_off[q] (device int64 array) or q * v_req_stride when v_req_off is NULL
 *   v_elems number of elements of the V allocation.  Every value read stays below it: the host
 *           checks strided layouts before launch (MR_ERR_INVALID_ARG); with a device offset table,
 *           a request whose rows do not fit inside [0, v_elems) (or, on the tensor-core kernel,
 *           whose offset is not a multiple of d_v) reads zeros instead and records
 *           MR_ERR_DEVICE_CHECK in the status word.  The tensor-core mixing kernel (bf16 maps of
 *           128-key blocks, at most 32 sender heads) also records MR_ERR_DEVICE_CHECK, writing no
 *           output, if the device places its dynamic shared memory off a 1024-byte boundary.
 *   O       output in dtype dt: element (q, r, i, c) at O + q * H_r * L * d_v + (r * L + i) * d_v + c
 *   opts    NULL or mr_retrieve_opts
 *   ws      workspace of at least mr_retrieve_workspace_bytes(map, H_r, d_v, n_req) bytes
 * Supported: d_v in {64, 128}; H_r <= 256.  bf16 maps with d_v = 128, block 64 or 128 and
 * H_s <= 64 run on the tensor-core kernel; other shapes on the CUDA-core kernel.  Within the
 * tensor-core kernel, bf16 maps of 128-key blocks with H_s <= 32 and n_req <= 1 mix the sender
 * heads on the tensor core too (weights rounded to bf16, fp32 accumulation); other maps mix them
 * on the CUDA cores (bf16 maps in fp32, fp8 maps in half precision).
 * Tiles a map could not store (capacity overflow at compression) contribute nothing and set
 * MR_ERR_CAPACITY in the status word.
 */
mr_status mr_retrieve(const mr_bsr* map, const float* W, int H_r, const void* V, int64_t v_elems,
                      void* O, mr_dtype dt, int d_v, int n_req, const int64_t* v_req_off,
                      int64_t v_req_stride, int64_t v_head_stride, const mr_retrieve_opts* opts,
                      void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes mr_dense_ref needs (device memory). */
size_t mr_dense_ref_workspace_bytes(int n_seq);

/*
 * Exact causal attention over packed variable-length sequences ("AttnCache Guide": the
 * standard softmax(QK^T * scale)V), with the same logit bias rule:
 *   Q [H][total_q][d], K [H][total_k][d], V [H][total_k][d_v], O [H][total_q][d_v] (dtype dt)
 *   cu_q, cu_k  device int32 [n_seq + 1] row offsets of each sequence in Q/O and K/V
 *   q_offset    device int32 [n_seq] absolute position of each sequence's first query row
 *               within its keys (NULL = 0): row i of sequence s attends keys
 *               0 .. q_offset[s] + i, and requires q_offset[s] + len_q(s) <= len_k(s)
 *   total_q, total_k  host ints equal to cu_q[n_seq] and cu_k[n_seq] (the per-head row
 *               counts of the packed tensors; total_q also sizes the launch)
 * Supported: d, d_v in {64, 128}.  bf16 with d = d_v = 128 (and per-key-block biases, if any, on
 * multiples of 32 keys) runs on the tensor-core kernel; other shapes on the CUDA-core kernel.
 * Requires q_offset[s] + len_q(s) <= len_k(s) (not checked: device arrays).
 */
mr_status mr_dense_ref(const void* Q, const void* K, const void* V, void* O, mr_dtype dt, int H,
                       int d, int d_v, const int32_t* cu_q, const int32_t* cu_k,
                       const int32_t* q_offset, int n_seq, int total_q, int total_k, float scale,
                       const mr_logit_bias* bias, void* ws, size_t ws_bytes, void* stream);

/*
 * Synchronise `stream` and return the device-side status recorded in `ws` (MR_OK if nothing
 * failed).  Every entry point that takes a workspace clears its status word when it is enqueued,
 * so the result describes the most recent call that used `ws`.
 */
mr_status mr_sync_status(void* ws, void* stream);

/* Synchronise `stream` and copy the map's kept-tile count to *nnz_host (host pointer). */
mr_status mr_bsr_nnz(const mr_bsr* map, int64_t* nnz_host, void* stream);

/*
 * Convert the first n_tiles tiles of map->vals to fp32 row-major tiles
 * ([n_tiles][block][block], element (a, b) = probability of query a on key b of the tile),
 * whatever the internal storage order.  out is device memory.
 */
mr_status mr_bsr_export(const mr_bsr* map, int64_t n_tiles, float* out, void* stream);

/*
 * Prefix-hash block manager: MapFlow section 5.3 ("Block Manager") and section 1 (prefix-hash
 * indexing).  Host-side index from token prefixes to stored compressed maps.
 *
 * Row (h, I) of a layer's map depends only on the first (I + 1) * block tokens (the map is
 * causal), so the maps stored for one sequence serve the first k query blocks of every request
 * whose first k * block tokens are the same: retrieve those rows with mr_retrieve's query-block
 * range and compute the rest.  Prefixes are keyed by a chained 64-bit hash per block of tokens
 * and checked token by token, so a hash collision is never reported as a hit.
 *
 * The manager keeps copies of the mr_bsr descriptors, never the device arrays: the caller keeps
 * an entry's arrays alive until the manager reports the entry evicted (mr_bm_evicted), and frees
 * them then.  Entries carry reference counts (the insert and each successful lookup take one;
 * mr_bm_release drops one).  When the bytes of the held entries exceed the budget, the least
 * recently used entries without references are evicted.  All calls are thread-safe, host-only,
 * and touch no device memory.
 */
typedef struct mr_block_manager mr_block_manager;

/* New manager for maps of `block`-token blocks; budget_bytes 0 = no limit.  NULL on bad
 * arguments or when host memory runs out. */
mr_block_manager* mr_bm_create(int block, int64_t budget_bytes);
void mr_bm_destroy(mr_block_manager* bm);

/*
 * Register the maps of one sequence: tokens (host int32 [n_tokens]; whole blocks are indexed, a
 * partial last block is ignored) and one descriptor per layer (host array of n_layers, each with
 * this block size and L >= the indexed tokens).  map_bytes is what the entry counts against the
 * budget.  Returns the entry id (>= 0, holding one reference) or -mr_status.
 */
int64_t mr_bm_insert(mr_block_manager* bm, const int32_t* tokens, int n_tokens, const mr_bsr* maps,
                     int n_layers, int64_t map_bytes);

/*
 * Longest stored prefix of `tokens` in whole blocks: returns k, the number of leading query blocks
 * whose map rows can be reused (0 = none), and writes the entry that holds them to *entry (-1 when
 * k = 0), taking a reference on it.  Negative -mr_status on bad arguments.
 */
int mr_bm_lookup(mr_block_manager* bm, const int32_t* tokens, int n_tokens, int64_t* entry);

/* Copy of the descriptor of `layer` of an entry. */
mr_status mr_bm_map(mr_block_manager* bm, int64_t entry, int layer, mr_bsr* out);

/* Drop one reference of an entry (then evict to the budget if needed). */
mr_status mr_bm_release(mr_block_manager* bm, int64_t entry);

/* Ids of evicted entries not reported yet (oldest first, at most max_ids): their device arrays are
 * no longer referenced by the manager.  Returns how many were written. */
int mr_bm_evicted(mr_block_manager* bm, int64_t* ids, int max_ids);

/* out[5] = {entries, bytes held, lookups, lookups that hit, query blocks served by hits}. */
mr_status mr_bm_stats(mr_block_manager* bm, int64_t* out);

/*
 * Measurement hooks (not part of the method).  When profiling is enabled, every entry point
 * records a CUDA event on its stream before and after each kernel it launches; mr_profile_read
 * waits for the recorded events and reports, per kernel id, the summed elapsed milliseconds and
 * the launch count since profiling was enabled.  Kernel ids are stable small integers; their
 * names come from mr_kernel_name (NULL past the last id).
 */
int mr_profile_enable(int on);      /* returns the previous state; enabling clears the records */
int mr_profile_read(double* total_ms, int64_t* launches, int max_ids); /* host arrays; returns ids */
const char* mr_kernel_name(int id);
int64_t mr_kernel_launches(void);   /* kernels launched by this library in this process */

/*
 * Measurement kernel (not part of the method): the retrieval's map reads alone.  Walks `map` in
 * the retrieval's order (128-row blocks longest first; key blocks J <= I; the kept tile of every
 * sender head) and moves each stored tile into shared memory `readers` times (by `readers` CTAs
 * working on the same row block side by side, as the retrieval's receiver-head groups do) with
 * 16-byte asynchronous copies, doing no arithmetic; each of its 512 threads keeps up to
 * ring_slots copies in flight (even, 2 .. 24).  Time it on `stream`; bytes moved =
 * readers * stored tiles * tile bytes.  ws: at least 256 bytes (status header).
 */
mr_status mr_gather_probe(const mr_bsr* map, int readers, int ring_slots, void* ws, size_t ws_bytes,
                          void* stream);

/*
 * Failure-path test hook (not part of the method; process-wide, for tests).  Sets the limit of the
 * tensor-core dense kernel's protocol waits to wait_ns (0 = the default 2 s; its softmax
 * warpgroups wait twice as long, so the wait nearest a stall reports it) and, with
 * skip_arrive = 1, makes the softmax warpgroup of each CTA's first query tile withhold its first
 * "P ready" arrive, so the MMA warp's wait runs out: the call records MR_ERR_TIMEOUT (detail
 * 0x913) in the workspace's status word, drains its copies and MMAs, frees Tensor Memory and
 * returns, leaving the context usable.
 * mr_debug_set(0, 0) restores normal operation.  No GPU fault is involved.
 */
mr_status mr_debug_set(uint64_t wait_ns, int skip_arrive);

#ifdef __cplusplus
}
#endif

#endif /* MR_H_ */
