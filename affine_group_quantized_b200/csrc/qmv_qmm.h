// qmv_qmm.h -- host interface of the many-row tensor-core kernel
// (qmv_qmm.cu), used by the C ABI in qmv_api.cu.  Internal to the library.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace qmvq {

// Activation rows per column block of a launch with M rows: 16, 32, 64 or 128.
int qmm_cols(int M);

// Codes of a weight row per pipeline stage: K must be a multiple.
int qmm_stage_codes(int bits);

// (weight tile, column block) tiles of a launch: ceil(N / 128) * ceil(M / cols).
long long qmm_tiles(int M, int N);

// Bytes of partial-sum scratch a launch on `sms` CTAs may use (split tiles).
size_t qmm_part_bytes(int M, int sms);

struct QmmArgs {
  const void *x;          // bf16 [M][K]
  const uint32_t *w;      // packed rows [N][K * bits / 32]
  const void *scales;     // bf16 [N][K / gs]
  const void *biases;     // bf16 [N][K / gs]
  void *y;                // bf16 [M][N]
  int M, N, K, bits, gs;
  int sms, smem_optin;
  int *err;               // status word: OR 2 when a bounded wait gives up
  float *part;            // partial-sum scratch (null: whole tiles per CTA)
  int *cnt;               // one zeroed counter per tile (null with part)
  cudaStream_t stream;
};

// Launch; returns 0 or a QMV_ERR_* code with a message in msg.
int qmm_launch(const QmmArgs &a, char *msg, size_t msg_len);

}  // namespace qmvq
