/*
 * oracle.c -- plain, slow, obviously-correct CPU reference for the affine
 * group-quantized matrix-vector product and its fused decode variants.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes
 * or calls this file; only the test suite, the package smoke check and the
 * CPU-baseline leg of the benchmark load it.  It shares no code, header,
 * table or helper with the CUDA path.
 *
 * Every result is computed in IEEE double precision, element by element, in
 * the order the definitions state.  No blocking, no reordering, no fusion.
 *
 * Sources (web pages, cited by page title and section):
 *   [MLX-Q]  "mlx/include/mlx/backend/metal/kernels/quantized.h" (MLX 0.30.1),
 *            pack factor / bytes-per-pack helpers, affine_dequantize kernel,
 *            qdot, adjust_matrix_offsets (gather form), affine_gather_qmm_rhs.
 *   [MLX-OPS] "Get trellis to run" compare page, mlx/ops.cpp
 *            extract_quantized_matmul_dims (shape rules).
 *   [GQMM]   "mlx.core.gather_qmm" API page (lhs_indices / rhs_indices,
 *            sorted_indices).
 *   [QW]     "QuantWeights" trait page and quant_weights.rs source page
 *            (gemv, gemv_gate_up_with, gemv_silu_gate, gemv_silu_gate_resid).
 *
 * Parity pins (what the self-tests check this file against) are listed at
 * each function.  All functions are pinned; none is "parity unpinned".
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "oracle.h"

/* ------------------------------------------------------------------------ */
/* Scalar helpers                                                            */
/* ------------------------------------------------------------------------ */

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
double oracle_bf16_to_double(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Valid bit widths and group sizes.
 * [MLX-Q] static_asserts in load_vector / qdot admit bits in {2,3,4,5,6,8};
 * the page's quantize/dequantize test sweeps group sizes {32, 64, 128}. */
static int bits_ok(int bits)
{
    return bits == 2 || bits == 3 || bits == 4 || bits == 5 || bits == 6 ||
           bits == 8;
}

static int gs_ok(int gs) { return gs == 32 || gs == 64 || gs == 128; }

/* Shape rule from [MLX-OPS] extract_quantized_matmul_dims: the packed row
 * holds K*bits/32 uint32 words and K/group_size groups.  We require K to be a
 * positive multiple of group_size, which makes K*bits a multiple of 32. */
int oracle_check_shape(int N, int K, int bits, int gs)
{
    if (N < 0 || K <= 0) return -1;
    if (!bits_ok(bits) || !gs_ok(gs)) return -1;
    if (K % gs != 0) return -1;
    if (((long long)K * bits) % 32 != 0) return -1;
    return 0;
}

/* Bytes in one packed row: K codes of `bits` bits, no padding. */
long long oracle_row_bytes(int K, int bits) { return (long long)K * bits / 8; }

/*
 * Code k of a packed row, read one bit at a time.
 *
 * Layout ([MLX-Q] affine_dequantize and the pack-factor helpers): the row is
 * one little-endian byte string; code k occupies bits [k*bits, (k+1)*bits) of
 * that string, least-significant bit first.  Pack boundaries (1 word for
 * 2/4/8 bits, 3 bytes for 3 and 6 bits, 5 bytes for 5 bits) all fall on byte
 * boundaries, so a single bitstream per row describes every width.
 */
static unsigned code_at(const uint8_t *row, long long k, int bits)
{
    unsigned q = 0;
    for (int b = 0; b < bits; ++b) {
        long long bit = k * bits + b;
        unsigned v = (row[bit >> 3] >> (bit & 7)) & 1u;
        q |= v << b;
    }
    return q;
}

/* Unpack all codes of an [N, K] packed matrix into one byte per code. */
int oracle_unpack(const uint32_t *w, int N, int K, int bits, uint8_t *codes)
{
    if (N < 0 || K <= 0 || !bits_ok(bits) || ((long long)K * bits) % 32 != 0)
        return -1;
    const long long rb = oracle_row_bytes(K, bits);
    const uint8_t *base = (const uint8_t *)w;
    for (long long n = 0; n < N; ++n)
        for (long long k = 0; k < K; ++k)
            codes[n * K + k] = (uint8_t)code_at(base + n * rb, k, bits);
    return 0;
}

/*
 * Dequantized weight: w_hat = scale * q + bias, with one (scale, bias) pair per
 * group_size consecutive codes of a row ([MLX-Q] affine_dequantize; qdot
 * returns scale*accum + sum*bias, the same affine map summed over a group).
 * In double this is exact: a bf16 times an integer below 256, plus a bf16.
 */
static double w_hat_at(const uint8_t *row, const uint16_t *srow,
                       const uint16_t *brow, long long k, int bits, int gs)
{
    double q = (double)code_at(row, k, bits);
    double s = oracle_bf16_to_double(srow[k / gs]);
    double b = oracle_bf16_to_double(brow[k / gs]);
    return s * q + b;
}

int oracle_dequant(const uint32_t *w, const uint16_t *scales,
                   const uint16_t *biases, int N, int K, int bits, int gs,
                   double *w_hat)
{
    if (oracle_check_shape(N, K, bits, gs)) return -1;
    const long long rb = oracle_row_bytes(K, bits);
    const long long G = K / gs;
    for (long long n = 0; n < N; ++n) {
        const uint8_t *row = (const uint8_t *)w + n * rb;
        for (long long k = 0; k < K; ++k)
            w_hat[n * K + k] =
                w_hat_at(row, scales + n * G, biases + n * G, k, bits, gs);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Row dot product: the definition y[m][n] = sum_k v[m][k] * w_hat[n][k]      */
/* ------------------------------------------------------------------------ */

/* One output: fp64 accumulation in k order; also the magnitude sum
 * A = sum_k |v_k * w_hat_k| that scales the acceptance tolerance. */
static void dot_row(const double *v, const uint8_t *row, const uint16_t *srow,
                    const uint16_t *brow, int K, int bits, int gs, double *y,
                    double *a)
{
    double acc = 0.0, mag = 0.0;
    for (long long k = 0; k < K; ++k) {
        double t = v[k] * w_hat_at(row, srow, brow, k, bits, gs);
        acc += t;
        mag += fabs(t);
    }
    *y = acc;
    *a = mag;
}

/* Work shared by the threaded drivers below.  v is the fp64 input vector
 * set [M][K]; out_rows lists which weight rows to evaluate (all when NULL). */
typedef struct {
    const double *v;
    const uint8_t *wbase;
    const uint16_t *s, *b;
    const int32_t *rows;
    int M, nrows, K, bits, gs;
    double *y, *a;
    int t, nt;
} job_t;

static void *job_run(void *p)
{
    job_t *j = (job_t *)p;
    const long long rb = oracle_row_bytes(j->K, j->bits);
    const long long G = j->K / j->gs;
    for (long long i = j->t; i < j->nrows; i += j->nt) {
        long long n = j->rows ? j->rows[i] : i;
        const uint8_t *row = j->wbase + n * rb;
        for (int m = 0; m < j->M; ++m)
            dot_row(j->v + (long long)m * j->K, row, j->s + n * G,
                    j->b + n * G, j->K, j->bits, j->gs,
                    j->y + (long long)m * j->nrows + i,
                    j->a + (long long)m * j->nrows + i);
    }
    return NULL;
}

static void run_jobs(job_t *proto, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads == 1) {
        proto->t = 0;
        proto->nt = 1;
        job_run(proto);
        return;
    }
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    job_t *js = (job_t *)malloc(sizeof(job_t) * nthreads);
    for (int t = 0; t < nthreads; ++t) {
        js[t] = *proto;
        js[t].t = t;
        js[t].nt = nthreads;
        pthread_create(&th[t], NULL, job_run, &js[t]);
    }
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
    free(js);
}

/*
 * qmv: y[m][n] = sum_k x[m][k] * w_hat[n][k]   (x @ dequant(W).T)
 *
 * [MLX-Q] qmv / qmv_fast (transpose = true), [QW] gemv ("decode matvec").
 * x is bf16 [M, K]; w is the packed [N, K] matrix; scales/biases bf16 [N, K/gs].
 * y and a are [M, nrows] (nrows = N when rows is NULL).
 *
 * Pins: brute force on tiny dyadic inputs (exact), the group-sum identity
 * sum_g scale_g*sum(x*q) + bias_g*sum(x), dense fp64 matmul of w_hat built
 * from known codes, bits=8 dense matmul.
 */
int oracle_qmv(const uint16_t *x, const uint32_t *w, const uint16_t *scales,
               const uint16_t *biases, int M, int N, int K, int bits, int gs,
               const int32_t *rows, int nrows, double *y, double *a,
               int nthreads)
{
    if (M < 0 || oracle_check_shape(N, K, bits, gs)) return -1;
    if (!rows) nrows = N;
    for (int i = 0; rows && i < nrows; ++i)
        if (rows[i] < 0 || rows[i] >= N) return -1;
    double *v = (double *)malloc(sizeof(double) * (size_t)M * K + 1);
    for (long long i = 0; i < (long long)M * K; ++i)
        v[i] = oracle_bf16_to_double(x[i]);
    job_t j = {v, (const uint8_t *)w, scales, biases, rows, M, nrows,
               K,  bits, gs, y, a, 0, 1};
    run_jobs(&j, nthreads);
    free(v);
    return 0;
}

/*
 * gate/up: gate_y = W_gate @ x and up_y = W_up @ x over ONE input x.
 * [QW] gemv_gate_up_with: two independent matvecs of the same shape; the
 * fused form only shares the read of x.  Pin: equals two qmv calls.
 */
int oracle_gate_up(const uint16_t *x, const uint32_t *wg, const uint16_t *sg,
                   const uint16_t *bg, const uint32_t *wu, const uint16_t *su,
                   const uint16_t *bu, int M, int N, int K, int bits, int gs,
                   double *yg, double *ag, double *yu, double *au,
                   int nthreads)
{
    if (oracle_qmv(x, wg, sg, bg, M, N, K, bits, gs, NULL, N, yg, ag,
                   nthreads))
        return -1;
    return oracle_qmv(x, wu, su, bu, M, N, K, bits, gs, NULL, N, yu, au,
                      nthreads);
}

/* silu(g) = g * sigmoid(g) = g / (1 + exp(-g)).  The pages name silu without
 * defining it; this is the standard definition. */
double oracle_silu(double g) { return g / (1.0 + exp(-g)); }

/*
 * silu-gate-resid:
 *   y[m][n] = x_resid[m][n] + sum_k w_hat[n][k] * (silu(gate[m][k]) * up[m][k])
 * [QW] gemv_silu_gate_resid (and gemv_silu_gate when x_resid is NULL).
 * gate, up: bf16 [M, K]; x_resid: bf16 [M, N] or NULL.  The gated input
 * silu(gate)*up is kept in fp64 (never rounded to bf16).  a[m][n] is the
 * magnitude sum of the matvec part only.
 * Pins: silu(g) - silu(-g) = g (odd-part identity), gate = 0 gives y = x_resid
 * exactly, composition with a dense fp64 matmul.
 */
int oracle_silu_gate_resid(const uint16_t *gate, const uint16_t *up,
                           const uint16_t *x_resid, const uint32_t *w,
                           const uint16_t *scales, const uint16_t *biases,
                           int M, int N, int K, int bits, int gs,
                           const int32_t *rows, int nrows, double *y,
                           double *a, int nthreads)
{
    if (M < 0 || oracle_check_shape(N, K, bits, gs)) return -1;
    if (!rows) nrows = N;
    for (int i = 0; rows && i < nrows; ++i)
        if (rows[i] < 0 || rows[i] >= N) return -1;
    double *v = (double *)malloc(sizeof(double) * (size_t)M * K + 1);
    for (long long i = 0; i < (long long)M * K; ++i)
        v[i] = oracle_silu(oracle_bf16_to_double(gate[i])) *
               oracle_bf16_to_double(up[i]);
    job_t j = {v, (const uint8_t *)w, scales, biases, rows, M, nrows,
               K,  bits, gs, y, a, 0, 1};
    run_jobs(&j, nthreads);
    free(v);
    if (x_resid) {
        for (int m = 0; m < M; ++m)
            for (int i = 0; i < nrows; ++i) {
                long long n = rows ? rows[i] : i;
                y[(long long)m * nrows + i] +=
                    oracle_bf16_to_double(x_resid[(long long)m * N + n]);
            }
    }
    return 0;
}

/*
 * gather: y[p] = x[lhs[p]] @ dequant(W[rhs[p]]).T  for p in [0, num_pairs).
 *
 * [MLX-Q] adjust_matrix_offsets (gather form) offsets x by lhs_indices[p] rows
 * and w/scales/biases by rhs_indices[p] experts; [GQMM] documents the flat
 * batch indices and that sorted_indices is only a performance hint, so the
 * value of every output row is the same whether or not the pairs are sorted.
 * lhs == NULL means pair p reads x row p.  Pairs whose index is out of range
 * are not computed; valid[p] is set to 0 for them (1 otherwise) and the
 * function returns how many there were.
 * x: bf16 [num_x_rows, K]; w: [E, N, K*bits/32] u32; scales/biases [E, N, K/gs];
 * y, a: [num_pairs, N].
 * Pins: equals qmv applied per pair; permuting pairs permutes rows.
 */
int oracle_gather(const uint16_t *x, const uint32_t *w, const uint16_t *scales,
                  const uint16_t *biases, const uint32_t *lhs,
                  const uint32_t *rhs, int num_pairs, int num_x_rows, int E,
                  int N, int K, int bits, int gs, double *y, double *a,
                  int32_t *valid, int nthreads)
{
    if (num_pairs < 0 || num_x_rows < 0 || E < 0 ||
        oracle_check_shape(N, K, bits, gs))
        return -1;
    const long long rb = oracle_row_bytes(K, bits);
    const long long G = K / gs;
    int bad = 0;
    for (int p = 0; p < num_pairs; ++p) {
        uint32_t xi = lhs ? lhs[p] : (uint32_t)p;
        uint32_t e = rhs[p];
        if (xi >= (uint32_t)num_x_rows || e >= (uint32_t)E) {
            valid[p] = 0;
            ++bad;
            continue;
        }
        valid[p] = 1;
        const uint8_t *wb = (const uint8_t *)w + (long long)e * N * rb;
        int rc = oracle_qmv(x + (long long)xi * K, (const uint32_t *)wb,
                            scales + (long long)e * N * G,
                            biases + (long long)e * N * G, 1, N, K, bits, gs,
                            NULL, N, y + (long long)p * N,
                            a + (long long)p * N, nthreads);
        if (rc) return -1;
    }
    return bad;
}
