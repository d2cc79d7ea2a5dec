// qmv_trellis.cuh -- the trellis-mode decode GEMV ("Get trellis to run"
// compare page, quantized.h: inst3 and qmv_trellis_impl).
//
//   y[m][n] = scale * sum_k x[m][k] * v(n, k),   scale = scales[0]
//
// Row n is W = K*bits/16 little-endian 16-bit words.  Value k = i*c + t
// (c = 16/bits values per word) has a 16-bit state made from word i (w0) and
// its successor w1 (word i+1; the row's last word is followed by its first):
// state 0 is w0; state t >= 1 takes its low bits*t bits from w1, with bit 0
// of that part flipped for odd t and bit `bits` flipped for t = 1.  The value
// of a state is the page's inst3: x = a*state + b in 32-bit arithmetic,
// keep the sign and low 12 bits of each half, XOR m, and add the two halves
// as binary16 numbers (one binary16 rounding).  There are no groups and no
// biases: one scale serves the matrix.
//
// A warp takes four or eight rows at a time; a lane takes chunks of 8 words
// (one 16-byte load per row) plus the word after them, so each word's
// successor is at hand.  The activation row sits in shared memory as fp32;
// a word's activations are read once (16-byte loads) for all the warp's
// rows.  Each value is a few integer
// and one binary16 operation away from its state; products and sums are
// fp32, reduced over the warp with shuffles, scaled and rounded once to
// bf16.
#pragma once

#include <cuda_fp16.h>

#include "qmv_device.cuh"

namespace qmvk {

constexpr int kTrellisWarps = 8;

struct TrellisParams {
  const uint16_t *w;       // rows of W 16-bit words
  const uint16_t *x;       // bf16 [M][K]
  const uint16_t *scales;  // bf16; scales[0] is the matrix scale
  uint16_t *y;             // bf16 [M][N]
  int M, N, K, W;          // W = K * bits / 16
};

// The page's inst3 with its default constants, for a 16-bit state.
__device__ __forceinline__ float trellis_value(uint32_t state) {
  uint32_t x = 89226354u * state + 64248484u;
  x = (x & 0x8FFF8FFFu) ^ 996162400u;
  __half2 h;
  *reinterpret_cast<uint32_t *>(&h) = x;
  return __half2float(__hadd(__low2half(h), __high2half(h)));
}

// Sum over the values of word w0 (successor w1), x from shared memory.
template <int BITS>
__device__ __forceinline__ float trellis_word(uint32_t w0, uint32_t w1, const float *xv) {
  constexpr int C = 16 / BITS;
  const uint32_t wx = w0 ^ w1;
  float acc = 0.f;
#pragma unroll
  for (int t = 0; t < C; ++t) {
    uint32_t s = w0;
    if (t > 0) {
      const uint32_t sel = (t & 1) ? (wx ^ 1u) : wx;
      s = w0 ^ (sel & ((1u << (BITS * t)) - 1u));
      if (t == 1) s ^= 1u << BITS;
    }
    acc = fmaf(xv[t], trellis_value(s & 0xFFFFu), acc);
  }
  return acc;
}

// Rows a warp works on at once: they share every activation load.
template <int BITS>
__host__ __device__ constexpr int trellis_rows_per_warp() { return BITS == 4 ? 8 : 4; }

template <int BITS>
__global__ void __launch_bounds__(kTrellisWarps * 32)
    qmv_trellis_kernel(const TrellisParams p) {
  extern __shared__ __align__(16) float xs[];  // the activation row, fp32 [K]
  constexpr int C = 16 / BITS;
  constexpr int RW = trellis_rows_per_warp<BITS>();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.y;
  grid_launch_dependents();
  grid_dependency_wait();
  for (int k = threadIdx.x; k < p.K; k += blockDim.x)
    xs[k] = bf16_to_f32(p.x[static_cast<size_t>(m) * p.K + k]);
  __syncthreads();
  const float scale = bf16_to_f32(p.scales[0]);
  const int nchunks = p.W / 8;  // 8-word chunks per row
  const int stride = gridDim.x * kTrellisWarps * RW;
  for (int n0 = (blockIdx.x * kTrellisWarps + warp) * RW; n0 < p.N; n0 += stride) {
    // RW rows (past N: row n0 again, its sums dropped)
    const uint16_t *row[RW];
#pragma unroll
    for (int r = 0; r < RW; ++r)
      row[r] = p.w + static_cast<size_t>(n0 + r < p.N ? n0 + r : n0) * p.W;
    float acc[RW];
#pragma unroll
    for (int r = 0; r < RW; ++r) acc[r] = 0.f;
    for (int ch = lane; ch < nchunks; ch += 32) {
      const int after = (8 * ch + 8) % p.W;  // the word after the chunk
      uint32_t u[RW][9];
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(row[r]) + ch);
        u[r][0] = v.x & 0xFFFFu;
        u[r][1] = v.x >> 16;
        u[r][2] = v.y & 0xFFFFu;
        u[r][3] = v.y >> 16;
        u[r][4] = v.z & 0xFFFFu;
        u[r][5] = v.z >> 16;
        u[r][6] = v.w & 0xFFFFu;
        u[r][7] = v.w >> 16;
        u[r][8] = __ldg(row[r] + after);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        // the word's C activations, read once for the RW rows
        float xv[C];
        const float4 *xp = reinterpret_cast<const float4 *>(xs + (8 * ch + i) * C);
#pragma unroll
        for (int q = 0; q < C / 4; ++q) {
          const float4 f = xp[q];
          xv[4 * q] = f.x;
          xv[4 * q + 1] = f.y;
          xv[4 * q + 2] = f.z;
          xv[4 * q + 3] = f.w;
        }
#pragma unroll
        for (int r = 0; r < RW; ++r) acc[r] += trellis_word<BITS>(u[r][i], u[r][i + 1], xv);
      }
    }
#pragma unroll
    for (int r = 0; r < RW; ++r) {
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int r = 0; r < RW; ++r)
        if (n0 + r < p.N) p.y[static_cast<size_t>(m) * p.N + n0 + r] = f32_to_bf16(scale * acc[r]);
    }
  }
}

}  // namespace qmvk
