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
 * The one exception is the quantizer, whose codes the pages decide in
 * binary32: it follows that precision operation by operation.
 *
 * Sources (web pages, cited by page title and section):
 *   [MLX-Q]  "mlx/include/mlx/backend/metal/kernels/quantized.h" (MLX 0.30.1),
 *            pack factor / bytes-per-pack helpers, affine_quantize and
 *            affine_dequantize kernels, qdot, adjust_matrix_offsets (gather
 *            form), affine_gather_qmm_rhs.
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

/* ------------------------------------------------------------------------ */
/* Producer side of the format: affine_quantize and affine_dequantize        */
/* ------------------------------------------------------------------------ */

/*
 * The bf16 value nearest to the exact sum hi + lo, ties to even, where hi and
 * lo are doubles with |lo| at most half an ulp of hi (the pair a two-sum
 * produces; lo == 0 for a single double).  bf16 keeps 8 significant bits and
 * the binary32 exponent range: below 2^-126 its spacing is fixed at 2^-133;
 * results of magnitude 2^128 and above overflow to infinity.
 *
 * hi is scaled by its bf16 spacing (a power of two, so exactly) and rounded
 * to an integer.  Because hi has at most 53 significant bits and lies on the
 * binary64 grid, the exact sum can only round differently from hi itself when
 * hi sits exactly halfway between two bf16 values; lo then decides.
 * Pins: brute force against exact rational rounding (ties, subnormals,
 * overflow included) in the test suite.
 */
uint16_t oracle_bf16_round(double hi, double lo)
{
    if (isnan(hi)) return 0x7fc0;
    if (isinf(hi)) return hi > 0 ? 0x7f80 : 0xff80;
    double r;
    if (hi == 0.0) {
        r = hi;
    } else {
        int e;
        frexp(hi, &e);                     /* 2^(e-1) <= |hi| < 2^e */
        int ue = e - 8 > -133 ? e - 8 : -133;
        double q = ldexp(hi, -ue);         /* exact */
        double fl = floor(q);
        double frac = q - fl;              /* exact */
        double n;
        if (frac > 0.5 || (frac == 0.5 && lo > 0.0)) n = fl + 1.0;
        else if (frac < 0.5 || (frac == 0.5 && lo < 0.0)) n = fl;
        else n = fmod(fl, 2.0) == 0.0 ? fl : fl + 1.0;   /* exact tie: even */
        r = ldexp(n, ue);
        if (r == 0.0) r = copysign(0.0, hi);
    }
    if (fabs(r) >= 0x1p128) return r > 0 ? 0x7f80 : 0xff80;
    float f = (float)r;                    /* exact: 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

static float bf16_to_float(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/*
 * Dequantize to bf16: out[n][k] = bf16(scale * q + bias), the affine map of
 * [MLX-Q] affine_dequantize, with the exact value rounded once to bf16 (ties
 * to even).  scale * q is exact in double (8 by 8 significant bits); the sum
 * with the bias is carried as a two-sum pair so the rounding is exact for any
 * exponents.
 * Pins: brute force with exact rationals; agreement with oracle_dequant
 * (the fp64 w_hat) wherever that is exact.
 */
int oracle_dequantize_bf16(const uint32_t *w, const uint16_t *scales,
                           const uint16_t *biases, int N, int K, int bits,
                           int gs, uint16_t *out)
{
    if (oracle_check_shape(N, K, bits, gs)) return -1;
    const long long rb = oracle_row_bytes(K, bits);
    const long long G = K / gs;
    for (long long n = 0; n < N; ++n) {
        const uint8_t *row = (const uint8_t *)w + n * rb;
        for (long long k = 0; k < K; ++k) {
            double a = oracle_bf16_to_double(scales[n * G + k / gs]) *
                       (double)code_at(row, k, bits);
            double b = oracle_bf16_to_double(biases[n * G + k / gs]);
            double s = a + b;              /* Knuth's two-sum: s + e == a + b */
            double bv = s - a;
            double av = s - bv;
            double e = (a - av) + (b - bv);
            out[n * K + k] = oracle_bf16_round(s, e);
        }
    }
    return 0;
}

/*
 * Quantize one group of gs weights, in binary32 as [MLX-Q] affine_quantize
 * computes it (the codes are decided in that precision):
 *   w_min starts at the largest finite bf16 and w_max at 0, then take the
 *   group's min and max (so w_max = max(0, max w));
 *   delta = max((w_max - w_min) / n_bins, 1e-7), n_bins = 2^bits - 1;
 *   the edge is the endpoint of larger magnitude (w_min when
 *   |w_min| > |w_max|, else w_max); the scale is +delta for the w_min edge
 *   and -delta for the w_max edge;
 *   q0 = round(edge / scale) (halves away from zero); unless q0 == 0 the scale
 *   becomes edge / q0 and the bias the edge itself (so the edge is code 0 and
 *   zero is code -q0), else the bias is 0;
 *   code = min(round((w - bias) / scale), n_bins).
 * scale and bias are stored as bf16 (round to nearest even); the codes use
 * the binary32 values.
 * Pins: hand-derived groups (tests/golden/quantize.txt); code 0 at the edge;
 * codes monotone in w; reconstruction within the rounding bound.
 */
static void quantize_group(const uint16_t *w, int gs, int bits, uint8_t *q,
                           uint16_t *scale_out, uint16_t *bias_out)
{
    const float n_bins = (float)((1 << bits) - 1);
    const float eps = 1e-7f;
    float w_min = bf16_to_float(0x7f7f);   /* largest finite bf16 */
    float w_max = 0.0f;
    for (int i = 0; i < gs; ++i) {
        float v = bf16_to_float(w[i]);
        w_min = fminf(w_min, v);
        w_max = fmaxf(w_max, v);
    }
    float scale = fmaxf((w_max - w_min) / n_bins, eps);
    int side = fabsf(w_min) > fabsf(w_max);
    scale = side ? scale : -scale;
    float edge = side ? w_min : w_max;
    float q0 = roundf(edge / scale);
    int at_zero = q0 == 0.0f;
    scale = at_zero ? scale : edge / q0;
    float bias = at_zero ? 0.0f : edge;
    *scale_out = oracle_bf16_round((double)scale, 0.0);
    *bias_out = oracle_bf16_round((double)bias, 0.0);
    for (int i = 0; i < gs; ++i) {
        float v = bf16_to_float(w[i]);
        float c = fminf(roundf((v - bias) / scale), n_bins);
        q[i] = (uint8_t)c;
    }
}

/* Write code k of a packed row, one bit at a time (the layout code_at reads). */
static void put_code(uint8_t *row, long long k, int bits, unsigned q)
{
    for (int b = 0; b < bits; ++b) {
        long long bit = k * bits + b;
        uint8_t m = (uint8_t)(1u << (bit & 7));
        if ((q >> b) & 1u) row[bit >> 3] |= m;
        else row[bit >> 3] &= (uint8_t)~m;
    }
}

/*
 * Quantize a bf16 [N, K] matrix: packed codes [N, K*bits/32] (the row layout
 * above), bf16 scales and biases [N, K/gs].  Groups are gs consecutive
 * elements of a row ([MLX-Q] affine_quantize indexes groups by element / gs
 * over the flattened matrix, which is the same thing when gs divides K).
 */
int oracle_affine_quantize(const uint16_t *w, int N, int K, int bits, int gs,
                           uint32_t *wq, uint16_t *scales, uint16_t *biases)
{
    if (oracle_check_shape(N, K, bits, gs)) return -1;
    const long long rb = oracle_row_bytes(K, bits);
    const long long G = K / gs;
    uint8_t q[128];
    for (long long n = 0; n < N; ++n) {
        uint8_t *row = (uint8_t *)wq + n * rb;
        for (long long g = 0; g < G; ++g) {
            quantize_group(w + n * K + g * gs, gs, bits, q, &scales[n * G + g],
                           &biases[n * G + g]);
            for (int i = 0; i < gs; ++i) put_code(row, g * gs + i, bits, q[i]);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* qvm: the product with the non-transposed matrix                            */
/* ------------------------------------------------------------------------ */

/*
 * qvm: y[m][n] = sum_k x[m][k] * w_hat[k][n]   (x @ dequant(W), transpose false)
 *
 * [MLX-Q] qvm_impl: the packed matrix has K rows (the input length) of N
 * codes (the output length), in the row layout above; its groups of gs run
 * along each row, so w_hat[k][n] = scales[k][n / gs] * q[k][n] +
 * biases[k][n / gs].  Each output sums its K terms in k order in fp64 and
 * records sum_k |x * w_hat|.
 * x bf16 [M, K]; w packed [K, N]; scales/biases bf16 [K, N/gs]; y, a [M, N].
 * Pins: a dense fp64 matmul of the dequantized matrix; brute force on
 * dyadic inputs (exact); equality with qmv of the transposed codes when the
 * scales are constant over each block of gs rows.
 */
int oracle_qvm(const uint16_t *x, const uint32_t *w, const uint16_t *scales,
               const uint16_t *biases, int M, int K, int N, int bits, int gs,
               double *y, double *a)
{
    if (M < 0 || oracle_check_shape(K, N, bits, gs)) return -1;
    const long long rb = oracle_row_bytes(N, bits);
    const long long G = N / gs;
    for (long long m = 0; m < M; ++m) {
        for (long long n = 0; n < N; ++n) {
            double acc = 0.0, mag = 0.0;
            for (long long k = 0; k < K; ++k) {
                const uint8_t *row = (const uint8_t *)w + k * rb;
                double t = oracle_bf16_to_double(x[m * K + k]) *
                           w_hat_at(row, scales + k * G, biases + k * G, n,
                                    bits, gs);
                acc += t;
                mag += fabs(t);
            }
            y[m * N + n] = acc;
            a[m * N + n] = mag;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Trellis mode ("Get trellis to run" compare page, quantized.h: inst3 and   */
/* qmv_trellis_impl)                                                         */
/* ------------------------------------------------------------------------ */

/* IEEE binary16 bit pattern -> double (exact). */
static double f16_to_double(uint16_t h)
{
    const int sign = h >> 15, e = (h >> 10) & 0x1F, m = h & 0x3FF;
    double v;
    if (e == 0) v = ldexp((double)m, -24);                 /* subnormal */
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(1024 + m), e - 25);            /* (1 + m/1024) 2^(e-15) */
    return sign ? -v : v;
}

/* The binary16 value nearest to v (ties to even), as a double.  v is the
 * exact sum of two binary16 values, so it is exact in double. */
static double round_to_f16(double v)
{
    if (v == 0.0 || isnan(v) || isinf(v)) return v;
    int e;
    frexp(fabs(v), &e);                /* 2^(e-1) <= |v| < 2^e */
    int ulp_exp = e - 11;              /* 11 significant bits */
    if (ulp_exp < -24) ulp_exp = -24;  /* subnormal spacing */
    const double n = nearbyint(ldexp(v, -ulp_exp));  /* default mode: ties to even */
    const double r = ldexp(n, ulp_exp);
    if (fabs(r) > 65504.0) return v > 0 ? INFINITY : -INFINITY;
    return r;
}

/* The value of a 16-bit trellis state (the page's inst3 with its default
 * constants a = 89226354, b = 64248484, m = 996162400): x = a * state + b in
 * 32-bit unsigned arithmetic, keep the sign bit and the low 12 bits of each
 * 16-bit half (mask 0x8FFF8FFF), XOR m, read the two halves as binary16
 * numbers and add them in binary16.
 * Pins: every state against an independent numpy float16 computation; a
 * hand-worked state (tests/golden/trellis.txt); the range of all values. */
double oracle_trellis_value(uint32_t state)
{
    uint32_t x = 89226354u * (state & 0xFFFFu) + 64248484u;
    x = (x & 0x8FFF8FFFu) ^ 996162400u;
    return round_to_f16(f16_to_double((uint16_t)(x & 0xFFFFu)) +
                        f16_to_double((uint16_t)(x >> 16)));
}

/* The state of value t (0 <= t < 16/bits) of word w0, whose successor word
 * is w1 (qmv_trellis_impl): t = 0 reads w0 itself; value t >= 1 takes its
 * low bits * t bits from w1 -- w0 ^ ((w0 ^ w1) & (2^(bits*t) - 1)) -- with
 * bit 0 of that part flipped for odd t, and bit `bits` flipped for t = 1.
 * Pins: the page's eight (2-bit) and four (4-bit) printed expressions, on
 * random word pairs. */
uint32_t oracle_trellis_state(uint32_t w0, uint32_t w1, int t, int bits)
{
    w0 &= 0xFFFFu;
    w1 &= 0xFFFFu;
    if (t == 0) return w0;
    const uint32_t wx = (w0 ^ w1) ^ ((t & 1) ? 1u : 0u);
    uint32_t s = w0 ^ (wx & ((1u << (bits * t)) - 1u));
    if (t == 1) s ^= 1u << bits;
    return s & 0xFFFFu;
}

/* Trellis-mode GEMV: y[m][n] = scale * sum_k x[m][k] * v(n, k), with scale
 * the first element of `scales` (the page's kernel reads scales[0]; biases
 * are not used), and a[m][n] = |scale| * sum_k |x[m][k] * v(n, k)|.
 * Row n is W = K*bits/16 little-endian 16-bit words u_0 .. u_{W-1}; value
 * k = i * (16/bits) + t has state oracle_trellis_state(u_i, u_{(i+1) mod W},
 * t, bits): the successor of the row's last word is its first word (the
 * reading of the page's successor word; see the design notes).
 * bits in {2, 4}; K * bits a multiple of 32 (rows of whole uint32 words).
 * Pins: a dense fp64 matmul of the value matrix built by the test's own
 * decoder; brute force on a tiny matrix with dyadic x. */
int oracle_qmv_trellis(const uint16_t *x, const uint32_t *w, const uint16_t *scales, int M,
                       int N, int K, int bits, double *y, double *a)
{
    if (M < 0 || N < 0 || K <= 0 || !(bits == 2 || bits == 4) || (K * bits) % 32 != 0)
        return -1;
    const long long W = (long long)K * bits / 16;
    const int cpw = 16 / bits;
    const double scale = oracle_bf16_to_double(scales[0]);
    for (long long n = 0; n < N; ++n) {
        const uint8_t *row = (const uint8_t *)w + n * W * 2;
        for (long long m = 0; m < M; ++m) {
            double acc = 0.0, mag = 0.0;
            for (long long i = 0; i < W; ++i) {
                const long long j = (i + 1) % W;
                const uint32_t w0 = row[2 * i] | ((uint32_t)row[2 * i + 1] << 8);
                const uint32_t w1 = row[2 * j] | ((uint32_t)row[2 * j + 1] << 8);
                for (int t = 0; t < cpw; ++t) {
                    const double v = oracle_trellis_value(oracle_trellis_state(w0, w1, t, bits));
                    const double p = oracle_bf16_to_double(x[m * K + i * cpw + t]) * v;
                    acc += p;
                    mag += fabs(p);
                }
            }
            y[m * N + n] = scale * acc;
            a[m * N + n] = fabs(scale) * mag;
        }
    }
    return 0;
}
