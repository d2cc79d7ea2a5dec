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
// Work units: the quantizer gives each lane a "chunk" of 8 consecutive codes
// of the flattened [N, K] matrix: 8 bf16 weights are one 16-byte load and 8
// codes of `bits` bits are exactly `bits` bytes of the packed stream (byte
// offset chunk * bits).  The dequantizer gives each thread "units" of 32
// codes: `bits` whole packed words in, 64 bytes of bf16 out.  Groups
// (group_size in {32, 64, 128}) are whole numbers of chunks and of units.
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

// The bf16 fused multiply-add computes s * q + b exactly and rounds once to
// bf16 (nearest, ties to even), which is the definition itself.  The code q
// enters as an exact bf16 value: for q < 128, the bits 0x4300 | q are the
// bf16 number 128 + q, and subtracting 128 is exact; 8-bit codes (up to 255)
// go through binary32 (0x4b000000 | q is 2^23 + q) and an exact conversion.
__device__ __forceinline__ __nv_bfloat162 bf162_bits(uint32_t v) {
  __nv_bfloat162 h;
  *reinterpret_cast<uint32_t *>(&h) = v;
  return h;
}
__device__ __forceinline__ uint32_t bf162_u32(__nv_bfloat162 h) {
  return *reinterpret_cast<uint32_t *>(&h);
}

// Dequantize works in units of 32 codes: exactly BITS packed words (4 * BITS
// bytes at a multiple of 4 * BITS, loaded with the widest aligned loads),
// always inside one group, and 64 bytes of bf16 output (four 16-byte
// stores).  Each thread takes two units per pass, both loaded before either
// is computed, so every thread keeps two loads in flight.
template <int BITS>
__device__ __forceinline__ void load_unit_words(const uint32_t *__restrict__ wq, long long u,
                                                uint32_t (&w)[BITS]) {
  const uint32_t *p = wq + u * BITS;
  if constexpr (BITS % 4 == 0) {
#pragma unroll
    for (int i = 0; i < BITS / 4; ++i) {
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p) + i);
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  } else if constexpr (BITS % 2 == 0) {
#pragma unroll
    for (int i = 0; i < BITS / 2; ++i) {
      const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p) + i);
      w[2 * i] = v.x; w[2 * i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < BITS; ++i) w[i] = __ldg(p + i);
  }
}

// Code i of a unit: bits [i * BITS, (i + 1) * BITS) of its little-endian
// stream, taken with a funnel shift where it straddles two words.
template <int BITS>
__device__ __forceinline__ uint32_t unit_code(const uint32_t (&w)[BITS], int i) {
  const int o = i * BITS, j = o >> 5, sh = o & 31;
  const uint32_t v = (sh + BITS > 32) ? __funnelshift_r(w[j], w[j + 1], sh) : (w[j] >> sh);
  return v & ((1u << BITS) - 1u);
}

// Codes 2j and 2j + 1 of a unit as an exact bf16 pair (code 2j low).
template <int BITS>
__device__ __forceinline__ __nv_bfloat162 code_pair(const uint32_t (&w)[BITS], int j) {
  const uint32_t c0 = unit_code<BITS>(w, 2 * j), c1 = unit_code<BITS>(w, 2 * j + 1);
  if constexpr (BITS == 8) {
    const float f0 = __fsub_rn(__uint_as_float(0x4b000000u | c0), 8388608.0f);
    const float f1 = __fsub_rn(__uint_as_float(0x4b000000u | c1), 8388608.0f);
    return __floats2bfloat162_rn(f0, f1);  // exact: integers below 256
  } else {
    return __hsub2(bf162_bits(c0 | (c1 << 16) | 0x43004300u), bf162_bits(0x43004300u));
  }
}

template <int BITS>
__device__ __forceinline__ void dequantize_unit(const uint32_t (&w)[BITS], uint32_t sb,
                                                uint32_t bb, uint4 *__restrict__ dst) {
  const __nv_bfloat162 s2 = bf162_bits(sb | (sb << 16)), b2 = bf162_bits(bb | (bb << 16));
#pragma unroll
  for (int c = 0; c < 4; ++c) {  // 8 codes per 16-byte store
    uint32_t h[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) h[j] = bf162_u32(__hfma2(code_pair<BITS>(w, 4 * c + j), s2, b2));
    dst[c] = make_uint4(h[0], h[1], h[2], h[3]);
  }
}

template <int BITS>
__global__ void __launch_bounds__(kThreads)
affine_dequantize_kernel(const uint32_t *__restrict__ wq,
                         const uint16_t *__restrict__ scales,
                         const uint16_t *__restrict__ biases,
                         uint4 *__restrict__ out, long long nunits,
                         int gs_shift) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long u0 = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
       u0 < nunits; u0 += 2 * stride) {
    const long long u1 = u0 + stride;
    const bool two = u1 < nunits;
    uint32_t w0[BITS], w1[BITS];
    load_unit_words<BITS>(wq, u0, w0);
    const long long g0 = (u0 * 32) >> gs_shift;
    const uint32_t s0 = __ldg(scales + g0), b0 = __ldg(biases + g0);
    uint32_t s1 = 0, b1 = 0;
    if (two) {
      load_unit_words<BITS>(wq, u1, w1);
      const long long g1 = (u1 * 32) >> gs_shift;
      s1 = __ldg(scales + g1);
      b1 = __ldg(biases + g1);
    }
    dequantize_unit<BITS>(w0, s0, b0, out + 4 * u0);
    if (two) dequantize_unit<BITS>(w1, s1, b1, out + 4 * u1);
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
// The code of one element: min(round(d / scale), n_bins) with the page's
// binary32 quotient d / scale and round-half-away.  The quotient is formed
// as d * (1 / scale) (both correctly rounded), within 3 * 2^-24 of the
// binary32 quotient relative to it; where no half-integer lies within
// 2^-20 * max(|t|, 1) of that product, both round to the same integer and
// rint gives it.  Only the rare elements near a half-integer take the IEEE
// division and roundf, so every code is the one the page's steps decide.
__device__ __forceinline__ uint32_t quantize_code(float v, float bias, float scale, float rcp,
                                                  float n_bins) {
  const float d = __fsub_rn(v, bias);
  const float tp = __fmul_rn(d, rcp);
  const float rt = rintf(tp);
  float code = rt;
  if (fabsf(__fsub_rn(tp, rt)) > 0.5f - fmaxf(fabsf(tp), 1.0f) * 0x1p-20f)
    code = roundf(__fdiv_rn(d, scale));
  return static_cast<uint32_t>(fminf(code, n_bins));
}

// The affine map of one group from its range [lo, hi] (lo taken from the
// largest finite bf16 down, hi from 0 up, as the page's affine_quantize
// starts them), in binary32 with IEEE divisions:
//   * the code step has magnitude max((hi - lo) / n_bins, 1e-7);
//   * the anchor is the endpoint of larger magnitude (hi on a tie); the step
//     takes the anchor's sign when the anchor is lo, the opposite sign when
//     it is hi, so codes grow away from the anchor into the range;
//   * the anchor's position on the code grid, j = round(anchor / step)
//     (halves away from zero), refines the step to anchor / j, and the
//     anchor becomes the offset -- unless j = 0, when the step stays and the
//     offset is 0.
// Returns the step (the stored scale) and the offset (the stored bias).
__device__ __forceinline__ float2 group_step_offset(float lo, float hi, float n_bins) {
  const float magnitude = fmaxf(__fdiv_rn(__fsub_rn(hi, lo), n_bins), 1e-7f);
  const bool anchor_is_lo = fabsf(lo) > fabsf(hi);
  const float anchor = anchor_is_lo ? lo : hi;
  const float step = anchor_is_lo ? magnitude : -magnitude;
  const float j = roundf(__fdiv_rn(anchor, step));
  if (j == 0.0f) return make_float2(step, 0.0f);
  return make_float2(__fdiv_rn(anchor, j), anchor);
}

// One work item: 32 chunks (one warp, lane = chunk).  Finds the group's
// range with xor butterflies over the group's lanes, stores the group's
// scale and bias from its first lane and the lane's packed codes.
template <int BITS, int GS>
__device__ __forceinline__ void quantize_item(const uint4 raw, long long c, bool live, int lane,
                                              uint8_t *__restrict__ wq,
                                              uint16_t *__restrict__ scales,
                                              uint16_t *__restrict__ biases) {
  constexpr int kLanes = GS / 8;  // lanes per group
  const float n_bins = static_cast<float>((1 << BITS) - 1);
  const float start_lo = bf16_bits_to_float(0x7f7fu);  // largest finite bf16
  const uint32_t pr[4] = {raw.x, raw.y, raw.z, raw.w};
  float v[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(pr[i] << 16);
    v[2 * i + 1] = __uint_as_float(pr[i] & 0xffff0000u);
  }
  float lo = start_lo, hi = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    lo = fminf(lo, v[i]);
    hi = fmaxf(hi, v[i]);
  }
#pragma unroll
  for (int o = 1; o < kLanes; o <<= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  const float2 so = group_step_offset(lo, hi, n_bins);
  const float scale = so.x, bias = so.y;
  if (live && (lane % kLanes) == 0) {
    const long long g = c / kLanes;
    scales[g] = __bfloat16_as_ushort(__float2bfloat16_rn(scale));
    biases[g] = __bfloat16_as_ushort(__float2bfloat16_rn(bias));
  }
  const float rcp = __frcp_rn(scale);
  uint64_t packed = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    packed |= static_cast<uint64_t>(quantize_code(v[i], bias, scale, rcp, n_bins)) << (BITS * i);
  if (live) store_chunk<BITS>(wq, c, packed);
}

// One lane per chunk; the GS / 8 lanes of a group are consecutive, and a
// work item's 32 chunks start on a group boundary, so the group's min and
// max are butterfly reductions inside those lanes.  All 32 lanes run every
// item (the loop bound is uniform over the warp); lanes past the end load
// nothing and store nothing, and since the chunk count is a whole number of
// groups they never share a group with a live lane.  A warp takes two items
// per pass (items wi and wi + warps), both loaded before either is computed.
template <int BITS, int GS>
__global__ void __launch_bounds__(kThreads)
affine_quantize_kernel(const uint4 *__restrict__ w, uint8_t *__restrict__ wq,
                       uint16_t *__restrict__ scales,
                       uint16_t *__restrict__ biases, long long nchunks) {
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
  const long long nwork = (nchunks + 31) / 32;
  for (long long wi = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + threadIdx.x / 32;
       wi < nwork; wi += 2 * warps) {
    const long long c0 = wi * 32 + lane, c1 = (wi + warps) * 32 + lane;
    const bool live0 = c0 < nchunks, live1 = c1 < nchunks;
    const bool item1 = wi + warps < nwork;  // warp-uniform
    uint4 r0 = make_uint4(0u, 0u, 0u, 0u), r1 = r0;
    if (live0) r0 = __ldg(w + c0);
    if (live1) r1 = __ldg(w + c1);
    quantize_item<BITS, GS>(r0, c0, live0, lane, wq, scales, biases);
    if (item1) quantize_item<BITS, GS>(r1, c1, live1, lane, wq, scales, biases);
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
  // one warp per two items of 32 chunks, kThreads / 32 warps per block
  int rc = launch_grid(((nchunks + 31) / 32 + 1) / 2, qmvq::kThreads / 32,
                       resident_blocks<kern>(), &grid);
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
  // two 32-code units per thread and pass
  const long long nunits = nchunks / 4;
  int rc = launch_grid((nunits + 1) / 2, qmvq::kThreads, resident_blocks<kern>(), &grid);
  if (rc) return rc;
  kern<<<grid, qmvq::kThreads, 0, st>>>(wq, s, b, out, nunits, gs_shift);
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
