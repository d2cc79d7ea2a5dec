/*
 * qmv.h -- C ABI of libqmv, the B200 (sm_100a) affine group-quantized
 * matrix-vector product and its fused decode variants.
 *
 * ---------------------------------------------------------------------------
 * Data format (shared by every entry point)
 * ---------------------------------------------------------------------------
 * A quantized weight W has N rows and K columns.  Each row is one packed,
 * unpadded bitstream of K codes of `bits` bits, least-significant bit first,
 * stored as K*bits/32 uint32 words (row byte stride K*bits/8).  Code k of a
 * row occupies bits [k*bits, (k+1)*bits) of the row's little-endian byte
 * string.  This is the layout of the pages' pack-factor helpers and
 * affine_dequantize kernel ("mlx/include/mlx/backend/metal/kernels/
 * quantized.h", MLX 0.30.1): 2/4/8-bit pack 16/8/4 codes per word, 3-bit 8
 * codes per 3 bytes, 5-bit 8 codes per 5 bytes, 6-bit 4 codes per 3 bytes.
 *
 * scales and biases are bf16 [N, K/group_size]; group g of row n covers
 * columns [g*group_size, (g+1)*group_size) and dequantizes as
 *     w_hat[n][k] = scale[n][g] * q[n][k] + bias[n][g]
 * (same page, affine_dequantize and qdot).  Scales may be negative.
 *
 * All activations and outputs are bf16 (passed as void*, uint16 bit
 * patterns), row-major and contiguous.  Arithmetic is fp32 with one final
 * round-to-nearest-even to bf16.
 *
 * Supported: bits in {2,3,4,5,6,8}; group_size in {32,64,128}; K a positive
 * multiple of group_size; N >= 1; M >= 1.
 *
 * ---------------------------------------------------------------------------
 * Conventions
 * ---------------------------------------------------------------------------
 * Pointers: every buffer pointer is a DEVICE pointer owned by the caller and
 * must be 16-byte aligned.  The library never frees or retains them.  It
 * allocates device memory in one place only: qmv's tensor-core path (several
 * activation rows) allocates its split-tile scratch on the first such call on
 * a device, and grows it when a call needs more; qmv_noalloc takes the same
 * operation without any allocation, and no other entry point allocates.
 * Streams: `stream` is a cudaStream_t (NULL = the legacy default stream).
 * Every call only enqueues work on that stream and returns; results are
 * ready when the stream is synchronized.  Each successful call enqueues one
 * kernel (qmv's tensor-core path also enqueues a clear of new scratch, on
 * the same stream, when it allocates).
 * Bounded waits: every wait inside the kernels gives up after a bound (a few
 * hundred milliseconds); a kernel whose wait gave up ORs 2 into a status
 * word -- gather_qmv's d_status when given, else the library's per-device
 * word that qmv_device_status reads -- and that launch's results are
 * undefined.  In a correct launch no wait comes near the bound.
 */
#ifndef LIBQMV_QMV_H
#define LIBQMV_QMV_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QMV_OK = 0,
    QMV_ERR_NULL = 1,        /* a required pointer is NULL                   */
    QMV_ERR_SHAPE = 2,       /* M, N, K, counts or group layout inconsistent */
    QMV_ERR_UNSUPPORTED = 3, /* bits / group_size outside the supported set  */
    QMV_ERR_ALIGN = 4,       /* a buffer pointer is not 16-byte aligned      */
    QMV_ERR_CUDA = 5         /* a CUDA runtime call or launch failed         */
} qmv_status;

/*
 * qmv -- y = x @ dequant(W).T
 *
 * Defined by the pages' quantized_matmul with transpose = true
 * ("mlx/include/mlx/backend/metal/kernels/quantized.h": qmv / qmv_fast) and
 * by the QuantWeights trait's gemv ("decode matvec y = self @ x").
 *   x       bf16 [M, K]
 *   w       uint32 [N, K*bits/32]  (packed rows, layout above)
 *   scales  bf16 [N, K/group_size]
 *   biases  bf16 [N, K/group_size]
 *   y       bf16 [M, N]  (written; must not overlap the inputs)
 *   y[m][n] = sum_k x[m][k] * w_hat[n][k]
 *
 * With 2-, 4- or 8-bit codes, K a multiple of 1024/bits and K/group_size a
 * multiple of 8, several activation rows run on the tensor cores:
 *   M = 3 .. 16: each w_hat is rounded once to fp16 and each x row is scaled
 *     by a power of two into fp16 range, with fp32 accumulation; scales and
 *     biases should lie in fp16's normal range (magnitude 2^-14 .. 65504);
 *   M >= 17 (the pages' qmm_t, "quantized.h": qmm_t_impl / affine_qmm_t):
 *     bf16 operands, w_hat = bf16(scale * q + bias) rounded once (the value
 *     dequantize writes), x as given, fp32 accumulation; blocks of 32, 64 or
 *     128 activation rows.
 * The first such call on a device allocates the paths' scratch (split-tile
 * partial sums: 2 x SMs x rows-per-block x 128 floats, at most 19.4 MB on a
 * 148-SM GPU, plus 4 bytes per tile); qmv_noalloc does the same without
 * allocating.
 */
int qmv(const void *x, const uint32_t *w, const void *scales,
        const void *biases, void *y, int M, int N, int K, int bits,
        int group_size, void *stream);

/*
 * qmv_noalloc -- the same operation, arguments and layouts as qmv, with no
 * device memory allocated by the library.  qmv's tensor-core path (several
 * activation rows, 2/4/8-bit codes) adds up 128-row tiles that are split
 * between CTAs through scratch memory the library allocates on first use;
 * for M = 3 .. 16 qmv_noalloc takes that scratch from a fixed array in the
 * library's device image instead (its address from cudaGetSymbolAddress, per
 * device), with results identical to qmv's; for M >= 17 it gives every CTA
 * whole tiles and needs no scratch at all (the same result within the
 * accuracy bound; the fp32 sums run in another order than qmv's).
 *   returns QMV_ERR_UNSUPPORTED when the call would need more than the array
 *   holds: more than 256 SMs, or more than 65536 row tiles (N > 8388608).
 * Calls on one device that use the array are expected in stream order.
 */
int qmv_noalloc(const void *x, const uint32_t *w, const void *scales,
                const void *biases, void *y, int M, int N, int K, int bits,
                int group_size, void *stream);

/*
 * qvm -- y = x @ dequant(W), the non-transposed product
 *
 * Defined by the pages' quantized_matmul with transpose = false
 * ("mlx/include/mlx/backend/metal/kernels/quantized.h": qvm_impl /
 * affine_qvm, the product the pages use for gradients).  W has K rows of N
 * codes each, in the packed row format above, and its groups run along N:
 *   x       bf16 [M, K]
 *   w       uint32 [K, N*bits/32]
 *   scales  bf16 [K, N/group_size]
 *   biases  bf16 [K, N/group_size]
 *   y       bf16 [M, N]  (written; must not overlap the inputs)
 *   y[m][n] = sum_k x[m][k] * (scale[k][n/gs] * q[k][n] + bias[k][n/gs])
 * N a positive multiple of group_size, K >= 1, 1 <= M <= 65535.  The rows
 * are split between the CTAs of a thread-block cluster (8, or 16 where the
 * device allows) whose partial sums are added in a fixed order
 * (deterministic results, no scratch memory).
 */
int qvm(const void *x, const uint32_t *w, const void *scales, const void *biases, void *y,
        int M, int K, int N, int bits, int group_size, void *stream);

/*
 * qmv_trellis -- trellis-mode GEMV: y = scale * x @ V.T
 *
 * Defined by the pages' trellis decode ("Get trellis to run" compare page,
 * quantized.h: inst3 and qmv_trellis_impl).  Row n of W is K*bits/16
 * little-endian 16-bit words (the packed row bytes read as uint16).  Value k
 * = i*(16/bits) + t of the row has a 16-bit state built from word i and its
 * successor word (word i+1; the row's last word is followed by its first):
 * t = 0 reads word i; t >= 1 takes the low bits*t bits from the successor,
 * with bit 0 of that part flipped for odd t and bit `bits` flipped for t = 1.
 * v(n, k) = inst3(state): x = 89226354*state + 64248484 (32-bit), keep the
 * sign and low 12 bits of each 16-bit half, XOR 996162400, and add the two
 * halves as binary16 numbers (one binary16 rounding).
 *   x       bf16 [M, K]
 *   w       uint32 [N, K*bits/32]
 *   scales  bf16; scales[0] scales the whole matrix (no groups, no biases)
 *   y       bf16 [M, N]  = bf16(scales[0] * sum_k x[m][k] * v(n, k)), fp32 sums
 * bits in {2, 4}; K*bits a multiple of 128, K <= 49152; 1 <= M <= 65535.
 */
int qmv_trellis(const void *x, const uint32_t *w, const void *scales, void *y, int M, int N,
                int K, int bits, void *stream);

/*
 * qmv_gate_up -- dual-output GEMV over one input, in ONE kernel launch:
 *   y_gate = x @ dequant(W_gate).T,   y_up = x @ dequant(W_up).T
 *
 * Defined by the QuantWeights trait's gemv_gate_up_with (pages
 * "QuantWeights" and "quant_weights.rs"): two matrices of the same shape
 * (the trait asserts equal in/out features), each with its own scales and
 * biases, one shared x.
 *   x                         bf16 [M, K]
 *   w_gate, w_up              uint32 [N, K*bits/32]
 *   s_gate, b_gate, s_up, b_up  bf16 [N, K/group_size]
 *   y_gate, y_up              bf16 [M, N]
 */
int qmv_gate_up(const void *x, const uint32_t *w_gate, const void *s_gate,
                const void *b_gate, const uint32_t *w_up, const void *s_up,
                const void *b_up, void *y_gate, void *y_up, int M, int N,
                int K, int bits, int group_size, void *stream);

/*
 * qmv_silu_gate_resid -- fused FFN tail with the residual add folded in:
 *   y[m][n] = x_resid[m][n] + sum_k w_hat[n][k] * silu(gate[m][k]) * up[m][k]
 *
 * Defined by the QuantWeights trait's gemv_silu_gate_resid; with
 * x_resid == NULL it is gemv_silu_gate (y = W @ (silu(gate) * up)).
 * silu(g) = g / (1 + exp(-g)).  silu(gate)*up is formed in fp32 inside the
 * kernel and is never rounded to bf16.
 *   gate, up   bf16 [M, K]
 *   x_resid    bf16 [M, N] or NULL
 *   w          uint32 [N, K*bits/32]; scales, biases bf16 [N, K/group_size]
 *   y          bf16 [M, N]
 */
int qmv_silu_gate_resid(const void *gate, const void *up, const void *x_resid,
                        const uint32_t *w, const void *scales,
                        const void *biases, void *y, int M, int N, int K,
                        int bits, int group_size, void *stream);

/*
 * gather_qmv -- index-gathered per-expert GEMV:
 *   y[p] = x[lhs_indices[p]] @ dequant(W[rhs_indices[p]]).T,  p < num_pairs
 *
 * Defined by the pages' gather_qmm ("mlx.core.gather_qmm": lhs_indices and
 * rhs_indices are flat indices into the batch dimensions of x and w;
 * sorted_indices "may allow a faster implementation") and by the gather
 * form of adjust_matrix_offsets in quantized.h.
 *   x            bf16 [num_x_rows, K]
 *   w            uint32 [num_experts, N, K*bits/32]
 *   scales/biases bf16 [num_experts, N, K/group_size]
 *   lhs_indices  uint32 [num_pairs] device array, or NULL (pair p reads x row p;
 *                then num_x_rows must be >= num_pairs)
 *   rhs_indices  uint32 [num_pairs] device array (expert of pair p)
 *   y            bf16 [num_pairs, N]
 *   sorted_indices  nonzero when rhs_indices is non-decreasing.  A hint
 *                only: the value of every output row is the same either way
 *                (bit-identical), whatever the order of the pairs.
 *   d_status     device int or NULL.  If any index is out of range the
 *                kernel ORs 1 into *d_status and leaves that pair's output
 *                row unwritten; valid pairs are still computed.  A bounded
 *                wait that gave up ORs 2 (see Conventions).  The caller
 *                zeroes *d_status before the call.
 * The kernel groups the pairs by expert itself (so sorting is only a hint)
 * and streams a touched expert's rows once per two of its pairs: an expert
 * with c pairs is read ceil(c / 2) times, its reads next to each other in
 * the launch so that the later ones mostly come from L2; untouched experts
 * are not read.  num_pairs may be 0 (nothing is enqueued).
 */
int gather_qmv(const void *x, const uint32_t *w, const void *scales,
               const void *biases, const uint32_t *lhs_indices,
               const uint32_t *rhs_indices, void *y, int num_pairs,
               int num_x_rows, int num_experts, int N, int K, int bits,
               int group_size, int sorted_indices, int *d_status,
               void *stream);

/*
 * affine_quantize -- quantize a bf16 matrix into the packed format above.
 *
 * Defined by the pages' affine_quantize kernel ("mlx/include/mlx/backend/
 * metal/kernels/quantized.h", MLX 0.30.1).  For each group of group_size
 * consecutive elements of a row, in binary32:
 *   w_min = min(largest finite bf16, group), w_max = max(0, group);
 *   delta = max((w_max - w_min) / n_bins, 1e-7), n_bins = 2^bits - 1;
 *   edge = w_min and scale = +delta if |w_min| > |w_max|,
 *   else edge = w_max and scale = -delta;
 *   q0 = round(edge / scale) (halves away from zero);
 *   if q0 != 0: scale = edge / q0, bias = edge; else bias = 0;
 *   code = min(round((w - bias) / scale), n_bins).
 * The codes are decided with the binary32 scale and bias; the stored scale
 * and bias are those values rounded to bf16 (nearest, ties to even), so the
 * bias is the group's edge exactly.  Every division is IEEE binary32
 * (correctly rounded), so codes, scales and biases are bit-identical to the
 * same steps run on any IEEE host.  Inputs must be finite; groups whose
 * values all lie within n_bins * 1e-7 of each other and exceed 1e31 in
 * magnitude overflow q0 and are outside the definition.
 *   w        bf16 [N, K] (read)
 *   w_q      uint32 [N, K*bits/32] (written; the row layout above)
 *   scales   bf16 [N, K/group_size] (written)
 *   biases   bf16 [N, K/group_size] (written)
 * N >= 0 (N = 0 enqueues nothing), K a positive multiple of group_size.
 * Outputs must not overlap the input.  One kernel launch; no allocation.
 * On error qmv_quant_last_error() describes the failure.
 */
int affine_quantize(const void *w, uint32_t *w_q, void *scales, void *biases,
                    int N, int K, int bits, int group_size, void *stream);

/*
 * affine_dequantize -- expand packed codes to bf16 weights:
 *   w_hat[n][k] = bf16(scale[n][g] * q[n][k] + bias[n][g]),  g = k / group_size
 *
 * Defined by the pages' affine_dequantize kernel (same page).  The exact value
 * scale * q + bias is rounded once to bf16 (nearest, ties to even), for any
 * scale and bias with |scale * q| < 2^128.
 *   w_q              uint32 [N, K*bits/32] (read; the row layout above)
 *   scales, biases   bf16 [N, K/group_size] (read)
 *   w_hat            bf16 [N, K] (written; must not overlap the inputs)
 * N >= 0 (N = 0 enqueues nothing), K a positive multiple of group_size.
 * One kernel launch; no allocation.  On error qmv_quant_last_error()
 * describes the failure.
 */
int affine_dequantize(const uint32_t *w_q, const void *scales,
                      const void *biases, void *w_hat, int N, int K, int bits,
                      int group_size, void *stream);

/* Message for the last non-OK return of affine_quantize or
 * affine_dequantize on this thread ("" if none). */
const char *qmv_quant_last_error(void);

/* Message for the last non-OK return of the other entry points on this
 * thread ("" if none). */
const char *qmv_last_error(void);

/* ABI version of this header (incremented on incompatible change). */
int qmv_abi_version(void);

/*
 * qmv_device_status -- read the current device's status word of the GEMV
 * kernels (no counterpart on the pages; part of this library's bounded-wait
 * error reporting, see Conventions).
 *   out     HOST int, written with the word: 0, or 2 if some kernel's
 *           bounded wait gave up since the last reset
 *   reset   nonzero: clear the word afterwards (enqueued on `stream`)
 *   stream  the word is read after the work already enqueued on `stream`;
 *           the call synchronizes that stream
 * Returns QMV_ERR_NULL for a NULL out, QMV_ERR_CUDA if a CUDA call fails.
 */
int qmv_device_status(int *out, int reset, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LIBQMV_QMV_H */
