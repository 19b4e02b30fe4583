/*
 * fp64 CPU oracle for cross-model attention-map reuse (MapFlow block top-p compression and
 * translated retrieval) and for exact causal attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code, header, table or helper with the
 * CUDA path: it is plain C, one row at a time, with no blocking, fusion or reordering beyond the
 * definitions it restates.
 *
 * Sources (page titles and sections):
 *   [MF]  "Accelerating Cross-Model LLM Inference via Attention Map Reuse"
 *         s2.1 (the attention map is the row softmax of scaled dot products),
 *         s3.3 (receiver heads are a non-negative normalised mix of sender heads),
 *         s4   (top-p compression into Block Sparse Row storage),
 *         s5.2 (block-level top-p in the Attention State Compressor),
 *         s5.4 (fused retrieval: translated map applied to the receiver's values).
 *   [AC]  "AttnCache Guide" section "The Quadratic Self-Attention Cost" (softmax(QK^T/sqrt(d_k))V).
 *
 * Readings of points the pages leave open (each is listed in the design notes):
 *   - scale sigma = 1/sqrt(d) of the sender head dim; logits s_ij = sigma q_i.k_j + b(h,i,j), j <= i;
 *   - b(h,i,j) is the MAXIMUM of the synthetic biases that apply to (i,j), 0 when none applies;
 *   - block mass M_IJ = (1/n_I) sum_{i in I} sum_{j in J} A_ij  (n_I = rows in block I), so
 *     sum_J M_IJ = 1;
 *   - selection: order J <= I by mass descending, ties to the smaller J; keep the first k blocks
 *     with k the least k >= 1 whose cumulative fp64 mass (in that order) is >= p; p >= 1 keeps all;
 *   - kept probabilities are stored as they are (no renormalisation); the renormalised variant
 *     divides each head's kept row by its kept mass (or_row_block_probs / or_retrieve_rows flag);
 *   - translated map  At_r[i,j] = sum_s W[r,s] A_s[i,j] [block(j) kept for (s, block(i))];
 *     output O_r[i] = sum_{j <= i} At_r[i,j] V_r[j].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_EXPORT __attribute__((visibility("default")))

typedef struct {
    int32_t sink_len;
    double sink_bias;
    int32_t window;
    double window_bias;
    const float* kb_bias; /* [H][n_kb], -inf = no bias on that key block; NULL = none */
    int32_t kb_block;
    int32_t n_kb;
} or_bias;

OR_EXPORT int or_version(void) { return 1; }

/* b(h, i, j): maximum of the applicable synthetic biases, 0 when none applies. */
static double bias_at(const or_bias* b, int h, int64_t i, int64_t j)
{
    int have = 0;
    double best = 0.0;
    if (b->sink_len > 0 && j < b->sink_len) {
        best = b->sink_bias;
        have = 1;
    }
    if (b->window > 0 && i - j < b->window) {
        if (!have || b->window_bias > best) best = b->window_bias;
        have = 1;
    }
    if (b->kb_bias != NULL) {
        int64_t jb = j / b->kb_block;
        if (jb < b->n_kb) {
            double v = (double)b->kb_bias[(int64_t)h * b->n_kb + jb];
            if (isfinite(v)) {
                if (!have || v > best) best = v;
                have = 1;
            }
        }
    }
    return have ? best : 0.0;
}

/*
 * One row of the causal attention map, [MF] s2.1 / [AC]:
 *   s_j = sigma * (q . k_j) + b(h, i_abs, j)  for j = 0 .. n_keys-1  (n_keys = i_abs + 1),
 *   out_j = exp(s_j - max s) / sum_j exp(s_j - max s).
 * Returns the natural-log normaliser  max s + log(sum exp(s - max s)).
 */
static double row_probs(const float* q, const float* Kh, int d, int64_t n_keys, double sigma,
                        const or_bias* b, int h, int64_t i_abs, double* out)
{
    double m = -INFINITY;
    for (int64_t j = 0; j < n_keys; ++j) {
        const float* k = Kh + j * d;
        double dot = 0.0;
        for (int t = 0; t < d; ++t) dot += (double)q[t] * (double)k[t];
        double s = sigma * dot + bias_at(b, h, i_abs, j);
        out[j] = s;
        if (s > m) m = s;
    }
    double l = 0.0;
    for (int64_t j = 0; j < n_keys; ++j) {
        out[j] = exp(out[j] - m);
        l += out[j];
    }
    for (int64_t j = 0; j < n_keys; ++j) out[j] /= l;
    return m + log(l);
}

/* Renormalised top-p row (the variant where the kept probabilities of a row are rescaled to sum
 * to 1; the pages leave renormalisation open): row[j] over keys j < n_keys of the row becomes
 * row[j] / sum_{j in kept blocks} row[j] for kept blocks and 0 elsewhere.  kept_row: [nKB] 0/1. */
static void renormalise_row(double* row, int64_t n_keys, const uint8_t* kept_row, int B)
{
    double m = 0.0;
    for (int64_t j = 0; j < n_keys; ++j)
        if (kept_row[j / B]) m += row[j];
    for (int64_t j = 0; j < n_keys; ++j) row[j] = (kept_row[j / B] && m > 0.0) ? row[j] / m : 0.0;
}

static void fill_bias(or_bias* b, int32_t sink_len, double sink_bias, int32_t window,
                      double window_bias, const float* kb_bias, int32_t kb_block, int32_t n_kb)
{
    b->sink_len = sink_len;
    b->sink_bias = sink_bias;
    b->window = window;
    b->window_bias = window_bias;
    b->kb_bias = kb_bias;
    b->kb_block = kb_block > 0 ? kb_block : 1;
    b->n_kb = n_kb;
}

/* ---------------------------------------------------------------------------------------------
 * Block top-p selection for one (layer, head, query-block) row of block masses, [MF] s4/s5.2.
 * mass[0..n-1] are the masses of the n causal key blocks.  Writes kept[J] = 1 for the kept
 * blocks, returns their count and the fp64 cumulative kept mass (summed in selection order).
 * ------------------------------------------------------------------------------------------- */
OR_EXPORT int or_select(const double* mass, int n, double p, uint8_t* kept, double* kept_mass)
{
    int* order = (int*)malloc(sizeof(int) * (size_t)(n > 0 ? n : 1));
    for (int t = 0; t < n; ++t) order[t] = t;
    /* insertion sort: larger mass first, equal masses -> smaller block index first */
    for (int a = 1; a < n; ++a) {
        int v = order[a];
        int c = a - 1;
        while (c >= 0 && (mass[order[c]] < mass[v] || (mass[order[c]] == mass[v] && order[c] > v))) {
            order[c + 1] = order[c];
            --c;
        }
        order[c + 1] = v;
    }
    int k = 0;
    double cum = 0.0;
    if (p >= 1.0) {
        for (k = 0; k < n; ++k) cum += mass[order[k]];
    } else {
        while (k < n) {
            cum += mass[order[k]];
            ++k;
            if (cum >= p) break;
        }
    }
    for (int t = 0; t < n; ++t) kept[t] = 0;
    for (int t = 0; t < k; ++t) kept[order[t]] = 1;
    if (kept_mass) *kept_mass = cum;
    free(order);
    return k;
}

/* ---------------------------------------------------------------------------------------------
 * Compression oracle, [MF] s4/s5.2: for each requested unit u = h * nQB + I compute the block
 * masses of query block I of head h, select the kept key blocks, and record per-row normalisers.
 *   Q, K     : [H][L][d] (dtype-rounded values, read as fp64)
 *   mass     : [H][nQB][nKB]  (entries J > I are 0)
 *   kept     : [H][nQB][nKB]  0/1
 *   count    : [H][nQB]
 *   kept_mass: [H][nQB]
 *   lse      : [H][L]  natural-log normaliser of each row (only rows of requested units)
 *   units    : list of unit ids, or NULL for all H*nQB units
 * ------------------------------------------------------------------------------------------- */
OR_EXPORT int or_compress(const float* Q, const float* K, int H, int L, int d, double sigma, double p,
                          int B, int32_t sink_len, double sink_bias, int32_t window,
                          double window_bias, const float* kb_bias, int32_t kb_block,
                          double* mass, uint8_t* kept, int32_t* count, double* kept_mass,
                          double* lse, const int32_t* units, int n_units, int n_threads)
{
    if (B <= 0 || L % B != 0) return 1;
    const int nQB = L / B, nKB = L / B;
    or_bias bias;
    fill_bias(&bias, sink_len, sink_bias, window, window_bias, kb_bias, kb_block,
              kb_bias ? L / (kb_block > 0 ? kb_block : 1) : 0);
    const int total = units ? n_units : H * nQB;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel
#endif
    {
        double* row = (double*)malloc(sizeof(double) * (size_t)L);
        double* m = (double*)malloc(sizeof(double) * (size_t)nKB);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int t = 0; t < total; ++t) {
            const int u = units ? units[t] : t;
            const int h = u / nQB, I = u % nQB;
            for (int J = 0; J < nKB; ++J) m[J] = 0.0;
            const int64_t i0 = (int64_t)I * B;
            for (int64_t i = i0; i < i0 + B; ++i) {
                const float* q = Q + ((int64_t)h * L + i) * d;
                double z = row_probs(q, K + (int64_t)h * L * d, d, i + 1, sigma, &bias, h, i, row);
                if (lse) lse[(int64_t)h * L + i] = z;
                for (int64_t j = 0; j <= i; ++j) m[j / B] += row[j];
            }
            for (int J = 0; J <= I; ++J) m[J] /= (double)B;
            double* mo = mass + (int64_t)u * nKB;
            for (int J = 0; J < nKB; ++J) mo[J] = (J <= I) ? m[J] : 0.0;
            uint8_t* ko = kept + (int64_t)u * nKB;
            memset(ko, 0, (size_t)nKB);
            double km = 0.0;
            count[u] = or_select(m, I + 1, p, ko, &km);
            kept_mass[u] = km;
        }
        free(m);
        free(row);
    }
    return 0;
}

/* Probabilities of one B x B tile (query block I, key block J) of head h; upper triangle of the
 * diagonal tile and the whole of tiles with J > I are 0.  out: [B][B]. */
OR_EXPORT int or_tile_probs(const float* Q, const float* K, int H, int L, int d, double sigma,
                            int B, int32_t sink_len, double sink_bias, int32_t window,
                            double window_bias, const float* kb_bias, int32_t kb_block, int h,
                            int I, int J, double* out)
{
    if (h < 0 || h >= H || B <= 0 || L % B) return 1;
    or_bias bias;
    fill_bias(&bias, sink_len, sink_bias, window, window_bias, kb_bias, kb_block,
              kb_bias ? L / (kb_block > 0 ? kb_block : 1) : 0);
    double* row = (double*)malloc(sizeof(double) * (size_t)L);
    for (int a = 0; a < B; ++a) {
        const int64_t i = (int64_t)I * B + a;
        row_probs(Q + ((int64_t)h * L + i) * d, K + (int64_t)h * L * d, d, i + 1, sigma, &bias,
                  h, i, row);
        for (int c = 0; c < B; ++c) {
            const int64_t j = (int64_t)J * B + c;
            out[a * B + c] = (j <= i) ? row[j] : 0.0;
        }
    }
    free(row);
    return 0;
}

/* Probabilities of every row of query block I of head h over all L keys, for a list of units
 * u = h * nQB + I: out[t][a][j] = A_h[I*B + a][j] for j <= I*B + a, else 0 ([MF] s2.1).  The rows are
 * the same softmax rows as or_tile_probs; this form returns a whole row block at once (a slab of
 * B x L) so that every stored tile of a unit can be checked without recomputing its rows.
 *   out : [n_units][B][L] */
OR_EXPORT int or_row_block_probs(const float* Q, const float* K, int H, int L, int d, double sigma,
                                 int B, int32_t sink_len, double sink_bias, int32_t window,
                                 double window_bias, const float* kb_bias, int32_t kb_block,
                                 const int32_t* units, int n_units, const uint8_t* kept, double* out,
                                 int n_threads)
{
    if (B <= 0 || L % B) return 1;
    const int nQB = L / B;
    for (int t = 0; t < n_units; ++t)
        if (units[t] < 0 || units[t] >= H * nQB) return 1;
    or_bias bias;
    fill_bias(&bias, sink_len, sink_bias, window, window_bias, kb_bias, kb_block,
              kb_bias ? L / (kb_block > 0 ? kb_block : 1) : 0);
    const int total = n_units * B;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 4)
#endif
    for (int x = 0; x < total; ++x) {
        const int t = x / B, a = x % B;
        const int h = units[t] / nQB, I = units[t] % nQB;
        const int64_t i = (int64_t)I * B + a;
        double* row = out + ((int64_t)t * B + a) * L;
        row_probs(Q + ((int64_t)h * L + i) * d, K + (int64_t)h * L * d, d, i + 1, sigma, &bias, h, i,
                  row);
        for (int64_t j = i + 1; j < L; ++j) row[j] = 0.0;
        if (kept) renormalise_row(row, i + 1, kept + ((int64_t)h * nQB + I) * nQB, B);
    }
    return 0;
}

/* ---------------------------------------------------------------------------------------------
 * Retrieval oracle, [MF] s3.3 + s5.4, evaluated on given kept sets (so selection and retrieval
 * can be checked separately):
 *   At_r[i,j] = sum_s W[r,s] * A_s[i,j] * kept[s][I(i)][J(j)],   O_r[i] = sum_{j<=i} At_r[i,j] V_r[j]
 * for each requested row i and each of n_req value sets.
 *   kept : [H_s][nQB][nKB] 0/1
 *   W    : [H_r][H_s]
 *   V    : request q at V + q * v_req_stride, laid out [H_r][L][dv]
 *   O    : [n_req][H_r][n_rows][dv]
 * ------------------------------------------------------------------------------------------- */
OR_EXPORT int or_retrieve_rows(const float* Q, const float* K, int H_s, int L, int d, double sigma,
                               int B, int32_t sink_len, double sink_bias, int32_t window,
                               double window_bias, const float* kb_bias, int32_t kb_block,
                               const uint8_t* kept, const float* W, int H_r, const float* V,
                               int n_req, int64_t v_req_stride, int dv, const int64_t* rows,
                               int n_rows, int renorm, double* O, int n_threads)
{
    if (B <= 0 || L % B) return 1;
    const int nQB = L / B, nKB = L / B;
    or_bias bias;
    fill_bias(&bias, sink_len, sink_bias, window, window_bias, kb_bias, kb_block,
              kb_bias ? L / (kb_block > 0 ? kb_block : 1) : 0);
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel
#endif
    {
        double* A = (double*)malloc(sizeof(double) * (size_t)H_s * (size_t)L);
        double* At = (double*)malloc(sizeof(double) * (size_t)L);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int t = 0; t < n_rows; ++t) {
            const int64_t i = rows[t];
            const int I = (int)(i / B);
            for (int s = 0; s < H_s; ++s) {
                double* a = A + (int64_t)s * L;
                row_probs(Q + ((int64_t)s * L + i) * d, K + (int64_t)s * L * d, d, i + 1, sigma,
                          &bias, s, i, a);
                const uint8_t* ks = kept + ((int64_t)s * nQB + I) * nKB;
                if (renorm) {
                    renormalise_row(a, i + 1, ks, B);
                } else {
                    for (int64_t j = 0; j <= i; ++j)
                        if (!ks[j / B]) a[j] = 0.0;
                }
            }
            for (int r = 0; r < H_r; ++r) {
                for (int64_t j = 0; j <= i; ++j) {
                    double acc = 0.0;
                    for (int s = 0; s < H_s; ++s) acc += (double)W[r * H_s + s] * A[(int64_t)s * L + j];
                    At[j] = acc;
                }
                for (int q = 0; q < n_req; ++q) {
                    const float* Vr = V + q * v_req_stride + (int64_t)r * L * dv;
                    double* o = O + (((int64_t)q * H_r + r) * n_rows + t) * dv;
                    for (int c = 0; c < dv; ++c) o[c] = 0.0;
                    for (int64_t j = 0; j <= i; ++j) {
                        const double w = At[j];
                        if (w == 0.0) continue;
                        const float* v = Vr + j * dv;
                        for (int c = 0; c < dv; ++c) o[c] += w * (double)v[c];
                    }
                }
            }
        }
        free(At);
        free(A);
    }
    return 0;
}

/* ---------------------------------------------------------------------------------------------
 * Exact causal attention for one sequence, [AC] formula, with the same logit bias rule:
 *   query row i (0 .. Lq-1) sits at absolute position q_offset + i and sees keys 0 .. q_offset+i.
 *   Q : [H][Lq][d], K : [H][Lk][d], V : [H][Lk][dv], O : [H][n_rows][dv]
 * ------------------------------------------------------------------------------------------- */
OR_EXPORT int or_dense_rows(const float* Q, const float* K, const float* V, int H, int Lq, int Lk,
                            int d, int dv, int64_t q_offset, double sigma, int32_t sink_len,
                            double sink_bias, int32_t window, double window_bias,
                            const float* kb_bias, int32_t kb_block, const int64_t* rows,
                            int n_rows, double* O, int n_threads)
{
    if (q_offset + Lq > Lk) return 1;
    or_bias bias;
    fill_bias(&bias, sink_len, sink_bias, window, window_bias, kb_bias, kb_block,
              kb_bias ? (Lk + (kb_block > 0 ? kb_block : 1) - 1) / (kb_block > 0 ? kb_block : 1) : 0);
    const int total = H * n_rows;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel
#endif
    {
        double* row = (double*)malloc(sizeof(double) * (size_t)Lk);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int u = 0; u < total; ++u) {
            const int h = u / n_rows, t = u % n_rows;
            const int64_t i = rows[t];
            const int64_t i_abs = q_offset + i;
            row_probs(Q + ((int64_t)h * Lq + i) * d, K + (int64_t)h * Lk * d, d, i_abs + 1, sigma,
                      &bias, h, i_abs, row);
            double* o = O + ((int64_t)h * n_rows + t) * dv;
            for (int c = 0; c < dv; ++c) o[c] = 0.0;
            for (int64_t j = 0; j <= i_abs; ++j) {
                const float* v = V + ((int64_t)h * Lk + j) * dv;
                for (int c = 0; c < dv; ++c) o[c] += row[j] * (double)v[c];
            }
        }
        free(row);
    }
    return 0;
}
