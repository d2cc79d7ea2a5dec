/*
 * oracle.h -- declarations of the plain CPU reference (oracle.c).
 * TEST INFRASTRUCTURE ONLY; never included by the product library.
 * All bf16 buffers are passed as uint16_t bit patterns; outputs are double.
 */
#ifndef QMV_ORACLE_H
#define QMV_ORACLE_H
#include <stdint.h>

double oracle_bf16_to_double(uint16_t h);
double oracle_silu(double g);
int oracle_check_shape(int N, int K, int bits, int gs);
long long oracle_row_bytes(int K, int bits);
int oracle_unpack(const uint32_t *w, int N, int K, int bits, uint8_t *codes);
int oracle_dequant(const uint32_t *w, const uint16_t *scales,
                   const uint16_t *biases, int N, int K, int bits, int gs,
                   double *w_hat);
int oracle_qmv(const uint16_t *x, const uint32_t *w, const uint16_t *scales,
               const uint16_t *biases, int M, int N, int K, int bits, int gs,
               const int32_t *rows, int nrows, double *y, double *a,
               int nthreads);
int oracle_gate_up(const uint16_t *x, const uint32_t *wg, const uint16_t *sg,
                   const uint16_t *bg, const uint32_t *wu, const uint16_t *su,
                   const uint16_t *bu, int M, int N, int K, int bits, int gs,
                   double *yg, double *ag, double *yu, double *au,
                   int nthreads);
int oracle_silu_gate_resid(const uint16_t *gate, const uint16_t *up,
                           const uint16_t *x_resid, const uint32_t *w,
                           const uint16_t *scales, const uint16_t *biases,
                           int M, int N, int K, int bits, int gs,
                           const int32_t *rows, int nrows, double *y,
                           double *a, int nthreads);
int oracle_gather(const uint16_t *x, const uint32_t *w, const uint16_t *scales,
                  const uint16_t *biases, const uint32_t *lhs,
                  const uint32_t *rhs, int num_pairs, int num_x_rows, int E,
                  int N, int K, int bits, int gs, double *y, double *a,
                  int32_t *valid, int nthreads);
uint16_t oracle_bf16_round(double hi, double lo);
int oracle_dequantize_bf16(const uint32_t *w, const uint16_t *scales,
                           const uint16_t *biases, int N, int K, int bits,
                           int gs, uint16_t *out);
int oracle_affine_quantize(const uint16_t *w, int N, int K, int bits, int gs,
                           uint32_t *wq, uint16_t *scales, uint16_t *biases);
int oracle_qvm(const uint16_t *x, const uint32_t *w, const uint16_t *scales,
               const uint16_t *biases, int M, int K, int N, int bits, int gs,
               double *y, double *a);
double oracle_trellis_value(uint32_t state);
uint32_t oracle_trellis_state(uint32_t w0, uint32_t w1, int t, int bits);
int oracle_qmv_trellis(const uint16_t *x, const uint32_t *w, const uint16_t *scales, int M,
                       int N, int K, int bits, double *y, double *a);
#endif
