// qmv_quant.cu -- the producer side of the packed format: affine_quantize
// (bf16 weights -> packed codes, bf16 scales and biases) and
// affine_dequantize (packed codes -> bf16 weights), kernels and C entry
// points.  Declarations and contracts are in include/qmv.h.
//
// Both operations follow the affine_quantize and affine_dequantize kernels of
// "mlx/include/mlx/backend/metal/kernels/quantized.h" (MLX 0.30.1).  Both are
// streaming, element-wise and HBM-bound (no contraction), so they run on the
// CUDA cores with 16-byte coalesced loads and stores and a grid-stride loop
// over one wave of resident blocks on every SM.
//
// Work unit: a "chunk" of 8 consecutive codes of the flattened [N, K]
// matrix.  8 codes of `bits` bits are exactly `bits` bytes of the packed
// stream (byte offset chunk * bits), and 8 bf16 weights are one 16-byte
// vector, so a chunk is the natural unit for both directions.  Groups
// (group_size in {32, 64, 128}) are whole numbers of chunks.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <string>

#include "qmv.h"

namespace qmvq {

constexpr int kThreads = 256;

__device__ __forceinline__ float bf16_bits_to_float(uint32_t h) {
  return __uint_as_float(h << 16);
}

// ---------------------------------------------------------------------------
// Dequantize: out = bf16(scale * q + bias), the exact value rounded once
// ---------------------------------------------------------------------------

// scale * q is exact in binary32 (8 by 8 significant bits), so one fused
// multiply-add rounds the exact scale * q + bias once to binary32 (r).  r
// rounds to bf16 exactly as the exact sum would, except when r lies exactly
// halfway between two bf16 values (its low 16 bits are 0x8000) while the sum
// was not exact: there the exact sum lies on the side of the two-sum error e,
// which the rare slow path recovers.
__device__ __noinline__ uint16_t affine_tie_to_bf16(float q, float s, float b, float r) {
  const float p = __fmul_rn(q, s);
  const float bv = __fsub_rn(r, p);
  const float av = __fsub_rn(r, bv);
  const float e = __fadd_rn(__fsub_rn(p, av), __fsub_rn(b, bv));
  const uint32_t u = __float_as_uint(r);
  if (e == 0.0f) return __bfloat16_as_ushort(__float2bfloat16_rn(r));  // a true tie
  // sign-magnitude: adding 1 to the upper half grows the magnitude
  const bool away = (e > 0.0f) == (r > 0.0f);
  return static_cast<uint16_t>((u >> 16) + (away ? 1u : 0u));
}

template <int BITS>
__global__ void __launch_bounds__(kThreads)
affine_dequantize_kernel(const uint32_t *__restrict__ wq,
                         const uint16_t *__restrict__ scales,
                         const uint16_t *__restrict__ biases,
                         uint4 *__restrict__ out, long long nchunks,
                         int gs_shift) {
  constexpr uint32_t kMask = (1u << BITS) - 1u;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long c = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
       c < nchunks; c += stride) {
    // the chunk's `BITS` bytes start at byte c * BITS; with at most 3 bytes
    // of offset into the first word they end within the next word
    const long long byte0 = c * BITS;
    const long long w0 = byte0 >> 2;
    const int off = static_cast<int>(byte0 & 3);
    uint64_t v = __ldg(wq + w0);
    if (off + BITS > 4) v |= static_cast<uint64_t>(__ldg(wq + w0 + 1)) << 32;
    v >>= 8 * off;
    const long long g = (c * 8) >> gs_shift;
    const float s = bf16_bits_to_float(__ldg(scales + g));
    const float b = bf16_bits_to_float(__ldg(biases + g));
    float q[8], r[8];
    bool tie = false;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      // the code as an exact float: 2^23 + q has q in its low mantissa bits
      const uint32_t code = static_cast<uint32_t>(v >> (BITS * i)) & kMask;
      q[i] = __fsub_rn(__uint_as_float(0x4b000000u | code), 8388608.0f);
      r[i] = __fmaf_rn(q[i], s, b);
      tie |= (__float_as_uint(r[i]) & 0xffffu) == 0x8000u;
    }
    uint32_t h[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat162 pr = __floats2bfloat162_rn(r[2 * j], r[2 * j + 1]);
      h[j] = *reinterpret_cast<const uint32_t *>(&pr);
    }
    if (tie) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if ((__float_as_uint(r[i]) & 0xffffu) == 0x8000u) {
          const uint32_t hi = affine_tie_to_bf16(q[i], s, b, r[i]);
          const int sh = 16 * (i & 1);
          h[i >> 1] = (h[i >> 1] & ~(0xffffu << sh)) | (hi << sh);
        }
      }
    }
    out[c] = make_uint4(h[0], h[1], h[2], h[3]);
  }
}

// ---------------------------------------------------------------------------
// Quantize: per group, the binary32 rules of the pages' affine_quantize
// ---------------------------------------------------------------------------

// Store the `BITS` packed bytes of chunk c (8 codes) at byte c * BITS.
template <int BITS>
__device__ __forceinline__ void store_chunk(uint8_t *wq, long long c, uint64_t p) {
  uint8_t *dst = wq + c * BITS;
  if constexpr (BITS == 2) {
    *reinterpret_cast<uint16_t *>(dst) = static_cast<uint16_t>(p);
  } else if constexpr (BITS == 4) {
    *reinterpret_cast<uint32_t *>(dst) = static_cast<uint32_t>(p);
  } else if constexpr (BITS == 8) {
    *reinterpret_cast<uint64_t *>(dst) = p;
  } else if constexpr (BITS == 6) {   // byte offset 6c is even
#pragma unroll
    for (int i = 0; i < 3; ++i)
      reinterpret_cast<uint16_t *>(dst)[i] = static_cast<uint16_t>(p >> (16 * i));
  } else {                            // 3 and 5: byte offsets of any alignment
#pragma unroll
    for (int i = 0; i < BITS; ++i) dst[i] = static_cast<uint8_t>(p >> (8 * i));
  }
}

// One lane per chunk; the GS / 8 lanes of a group are consecutive, and a
// warp's 32 chunks start on a group boundary, so the group's min and max are
// butterfly reductions inside those lanes.  All 32 lanes run every
// iteration (the loop bound is uniform over the warp); lanes past the end
// load nothing and store nothing, and since the chunk count is a whole number
// of groups they never share a group with a live lane.
template <int BITS, int GS>
__global__ void __launch_bounds__(kThreads)
affine_quantize_kernel(const uint4 *__restrict__ w, uint8_t *__restrict__ wq,
                       uint16_t *__restrict__ scales,
                       uint16_t *__restrict__ biases, long long nchunks) {
  constexpr int kLanes = GS / 8;  // lanes per group
  const float n_bins = static_cast<float>((1 << BITS) - 1);
  const float eps = 1e-7f;
  const float start_min = bf16_bits_to_float(0x7f7fu);  // largest finite bf16
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
  const long long nwork = (nchunks + 31) / 32;
  for (long long wi = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
       wi < nwork; wi += warps) {
    const long long c = wi * 32 + lane;
    const bool live = c < nchunks;
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    if (live) raw = __ldg(w + c);
    const uint32_t pr[4] = {raw.x, raw.y, raw.z, raw.w};
    float v[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(pr[i] << 16);
      v[2 * i + 1] = __uint_as_float(pr[i] & 0xffff0000u);
    }
    float w_min = start_min, w_max = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      w_min = fminf(w_min, v[i]);
      w_max = fmaxf(w_max, v[i]);
    }
#pragma unroll
    for (int o = 1; o < kLanes; o <<= 1) {
      w_min = fminf(w_min, __shfl_xor_sync(0xffffffffu, w_min, o));
      w_max = fmaxf(w_max, __shfl_xor_sync(0xffffffffu, w_max, o));
    }
    float scale = fmaxf(__fdiv_rn(__fsub_rn(w_max, w_min), n_bins), eps);
    const bool side = fabsf(w_min) > fabsf(w_max);
    scale = side ? scale : -scale;
    const float edge = side ? w_min : w_max;
    const float q0 = roundf(__fdiv_rn(edge, scale));
    const bool at_zero = q0 == 0.0f;
    scale = at_zero ? scale : __fdiv_rn(edge, q0);
    const float bias = at_zero ? 0.0f : edge;
    if (live && (lane % kLanes) == 0) {
      const long long g = c / kLanes;
      scales[g] = __bfloat16_as_ushort(__float2bfloat16_rn(scale));
      biases[g] = __bfloat16_as_ushort(__float2bfloat16_rn(bias));
    }
    uint64_t packed = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float t = __fdiv_rn(__fsub_rn(v[i], bias), scale);
      const uint32_t q = static_cast<uint32_t>(fminf(roundf(t), n_bins));
      packed |= static_cast<uint64_t>(q) << (BITS * i);
    }
    if (live) store_chunk<BITS>(wq, c, packed);
  }
}

}  // namespace qmvq

// ---------------------------------------------------------------------------
// C entry points
// ---------------------------------------------------------------------------

namespace {

thread_local std::string g_quant_error;

int qfail(int code, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
int qfail(int code, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_quant_error = buf;
  return code;
}

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_quant_shape(int N, int K, int bits, int gs) {
  if (bits != 2 && bits != 3 && bits != 4 && bits != 5 && bits != 6 && bits != 8)
    return qfail(QMV_ERR_UNSUPPORTED, "bits=%d is not one of 2,3,4,5,6,8", bits);
  if (gs != 32 && gs != 64 && gs != 128)
    return qfail(QMV_ERR_UNSUPPORTED, "group_size=%d is not one of 32,64,128", gs);
  if (N < 0 || K <= 0)
    return qfail(QMV_ERR_SHAPE, "N=%d, K=%d: need N >= 0 and K >= 1", N, K);
  if (K % gs != 0)
    return qfail(QMV_ERR_SHAPE, "K=%d is not a multiple of group_size=%d", K, gs);
  return QMV_OK;
}

// Blocks of kernel `Kern` that fit on one SM at kThreads threads (its
// registers decide it), asked once per kernel.
template <auto Kern>
int resident_blocks() {
  static const int n = [] {
    int b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, Kern, qmvq::kThreads, 0) !=
            cudaSuccess ||
        b < 1)
      b = 1;
    return b;
  }();
  return n;
}

// Grid of the grid-stride loops: one full wave (resident blocks x SMs), or
// fewer blocks when there is less work.
int launch_grid(long long items, int items_per_block, int per_sm, int *grid) {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return qfail(QMV_ERR_CUDA, "no usable CUDA device");
  const long long cap = static_cast<long long>(sms) * per_sm;
  const long long need = (items + items_per_block - 1) / items_per_block;
  *grid = static_cast<int>(need < cap ? need : cap);
  return QMV_OK;
}

template <int BITS, int GS>
int launch_quantize_gs(cudaStream_t st, const uint4 *w, uint8_t *wq, uint16_t *s,
                       uint16_t *b, long long nchunks) {
  constexpr auto kern = qmvq::affine_quantize_kernel<BITS, GS>;
  int grid = 0;
  // one warp per 32 chunks, kThreads / 32 warps per block
  int rc = launch_grid((nchunks + 31) / 32, qmvq::kThreads / 32, resident_blocks<kern>(), &grid);
  if (rc) return rc;
  kern<<<grid, qmvq::kThreads, 0, st>>>(w, wq, s, b, nchunks);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return qfail(QMV_ERR_CUDA, "affine_quantize launch: %s", cudaGetErrorString(e));
  return QMV_OK;
}

template <int BITS>
int launch_quantize(int gs, cudaStream_t st, const uint4 *w, uint8_t *wq, uint16_t *s,
                    uint16_t *b, long long nchunks) {
  if (gs == 32) return launch_quantize_gs<BITS, 32>(st, w, wq, s, b, nchunks);
  if (gs == 64) return launch_quantize_gs<BITS, 64>(st, w, wq, s, b, nchunks);
  return launch_quantize_gs<BITS, 128>(st, w, wq, s, b, nchunks);
}

template <int BITS>
int launch_dequantize(int gs_shift, cudaStream_t st, const uint32_t *wq, const uint16_t *s,
                      const uint16_t *b, uint4 *out, long long nchunks) {
  constexpr auto kern = qmvq::affine_dequantize_kernel<BITS>;
  int grid = 0;
  int rc = launch_grid(nchunks, qmvq::kThreads, resident_blocks<kern>(), &grid);
  if (rc) return rc;
  kern<<<grid, qmvq::kThreads, 0, st>>>(wq, s, b, out, nchunks, gs_shift);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return qfail(QMV_ERR_CUDA, "affine_dequantize launch: %s", cudaGetErrorString(e));
  return QMV_OK;
}

}  // namespace

extern "C" {

int affine_quantize(const void *w, uint32_t *w_q, void *scales, void *biases, int N,
                    int K, int bits, int group_size, void *stream) {
  if (!w || !w_q || !scales || !biases)
    return qfail(QMV_ERR_NULL, "w, w_q, scales and biases must not be NULL");
  int rc = check_quant_shape(N, K, bits, group_size);
  if (rc) return rc;
  if (!al16(w) || !al16(w_q) || !al16(scales) || !al16(biases))
    return qfail(QMV_ERR_ALIGN, "every buffer must be 16-byte aligned");
  g_quant_error.clear();
  const long long nchunks = static_cast<long long>(N) * K / 8;
  if (nchunks == 0) return QMV_OK;
  auto st = static_cast<cudaStream_t>(stream);
  auto wv = static_cast<const uint4 *>(w);
  auto qb = reinterpret_cast<uint8_t *>(w_q);
  auto s = static_cast<uint16_t *>(scales);
  auto b = static_cast<uint16_t *>(biases);
  switch (bits) {
    case 2: return launch_quantize<2>(group_size, st, wv, qb, s, b, nchunks);
    case 3: return launch_quantize<3>(group_size, st, wv, qb, s, b, nchunks);
    case 4: return launch_quantize<4>(group_size, st, wv, qb, s, b, nchunks);
    case 5: return launch_quantize<5>(group_size, st, wv, qb, s, b, nchunks);
    case 6: return launch_quantize<6>(group_size, st, wv, qb, s, b, nchunks);
    default: return launch_quantize<8>(group_size, st, wv, qb, s, b, nchunks);
  }
}

int affine_dequantize(const uint32_t *w_q, const void *scales, const void *biases,
                      void *w_hat, int N, int K, int bits, int group_size, void *stream) {
  if (!w_q || !scales || !biases || !w_hat)
    return qfail(QMV_ERR_NULL, "w_q, scales, biases and w_hat must not be NULL");
  int rc = check_quant_shape(N, K, bits, group_size);
  if (rc) return rc;
  if (!al16(w_q) || !al16(scales) || !al16(biases) || !al16(w_hat))
    return qfail(QMV_ERR_ALIGN, "every buffer must be 16-byte aligned");
  g_quant_error.clear();
  const long long nchunks = static_cast<long long>(N) * K / 8;
  if (nchunks == 0) return QMV_OK;
  const int gs_shift = group_size == 32 ? 5 : group_size == 64 ? 6 : 7;
  auto st = static_cast<cudaStream_t>(stream);
  auto s = static_cast<const uint16_t *>(scales);
  auto b = static_cast<const uint16_t *>(biases);
  auto out = static_cast<uint4 *>(w_hat);
  switch (bits) {
    case 2: return launch_dequantize<2>(gs_shift, st, w_q, s, b, out, nchunks);
    case 3: return launch_dequantize<3>(gs_shift, st, w_q, s, b, out, nchunks);
    case 4: return launch_dequantize<4>(gs_shift, st, w_q, s, b, out, nchunks);
    case 5: return launch_dequantize<5>(gs_shift, st, w_q, s, b, out, nchunks);
    case 6: return launch_dequantize<6>(gs_shift, st, w_q, s, b, out, nchunks);
    default: return launch_dequantize<8>(gs_shift, st, w_q, s, b, out, nchunks);
  }
}

const char *qmv_quant_last_error(void) { return g_quant_error.c_str(); }

}  // extern "C"
