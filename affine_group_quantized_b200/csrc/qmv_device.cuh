// qmv_device.cuh -- device building blocks for the sm_100a quantized GEMV
// kernels: mbarrier / bulk-copy wrappers, the per-bit-width code decoder and
// the bf16 helpers.  Everything here is written for this library from the
// PTX ISA and the IEEE-754 binary32 definition.
#pragma once

#include <cstdint>
#include <utility>

#include <cuda_bf16.h>

namespace qmvk {

// ---------------------------------------------------------------------------
// Shared-memory addresses, mbarriers, bulk copies
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)),
               "r"(count)
               : "memory");
}

// Make barrier initialisation visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// One arrival that also announces `bytes` of incoming bulk-copy data.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar,
                                                      uint32_t bytes) {
  asm volatile(
      "mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  Every wait
// in these kernels is on copies the same CTA issued, so it ends unless a copy
// faulted; the bound only keeps a broken launch from spinning for ever.
// Returns false when the bound is hit.
constexpr uint32_t kWaitLimit = 1u << 22;  // try_wait rounds (each may suspend)

__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitLimit; ++i)
    if (mbar_test(bar, parity)) return true;
  return false;
}

// 1-D bulk copy global -> shared, completing `bytes` on `bar`.  Both
// addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src,
                                         uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];\n" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Named barrier over the first `nthreads` threads (a multiple of 32).
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// bf16 / binary32 helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ float bf16_to_f32(uint16_t h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}

__device__ __forceinline__ uint16_t f32_to_bf16(float v) {
  __nv_bfloat16 b = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t *>(&b);
}

// 2^e for e in [-126, 127], built from the exponent field.
__device__ __forceinline__ float pow2i(int e) {
  return __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
}

// ---------------------------------------------------------------------------
// Code decoder
//
// A "unit" is 32 consecutive codes of a row: exactly `BITS` 32-bit words,
// and always inside one quantization group (group sizes are multiples of 32).
// Code i of the unit sits at bits [i*BITS, (i+1)*BITS) of the unit's
// little-endian bitstream.
//
// Each code is turned into a binary32 with ONE bitwise AND: the AND keeps the
// code's bits at some position p <= 23-BITS inside the fraction field of a
// 32-bit "view" of the stream, and leaves the exponent field zero, so the
// float is the subnormal q * 2^(p-149) exactly.  A view is either a stream
// word itself (free) or a funnel shift of two adjacent words (one
// instruction, shared by every code it covers).  The position p of each code
// is a compile-time constant; the matching activation is pre-multiplied by
// 2^(149-p-c), so x'' * f = x * q * 2^-c exactly (the product of a bf16 and an
// integer below 256 has at most 16 significant bits).  c is chosen per unit
// from the unit's largest |x| so nothing overflows; the unit's partial sum is
// scaled back by 2^c before the group scale is applied.
// ---------------------------------------------------------------------------

// Bit offset (from the start of the unit) of the view that holds code i.
// Greedy: use the word-aligned view when the code fits inside its low 23
// bits, else the most recent shifted view if it still covers the code, else
// open a new shifted view starting at the code.
__host__ __device__ constexpr int view_offset(int bits, int i) {
  int cur = -1;
  int o = 0;
  for (int j = 0; j <= i; ++j) {
    const int a = j * bits;
    const int wa = (a / 32) * 32;
    if (a - wa + bits <= 23) {
      o = wa;
    } else if (cur >= 0 && a >= cur && a - cur + bits <= 23) {
      o = cur;
    } else {
      cur = a;
      o = a;
    }
  }
  return o;
}

__host__ __device__ constexpr int code_pos(int bits, int i) {
  return i * bits - view_offset(bits, i);
}

template <int BITS, int I>
__device__ __forceinline__ float code_as_float(const uint32_t (&wd)[BITS]) {
  constexpr int o = view_offset(BITS, I);
  constexpr int p = I * BITS - o;
  constexpr int wi = o / 32;
  constexpr int sh = o % 32;
  static_assert(p >= 0 && p + BITS <= 23, "code outside fraction field");
  uint32_t v;
  if constexpr (sh == 0) {
    v = wd[wi];
  } else if constexpr (wi + 1 < BITS) {
    v = __funnelshift_r(wd[wi], wd[wi + 1], sh);
  } else {
    v = wd[wi] >> sh;
  }
  constexpr uint32_t mask = ((1u << BITS) - 1u) << p;
  return __uint_as_float(v & mask);
}

template <int BITS, int MR, int J>
__device__ __forceinline__ void fma_code_pair(const uint32_t (&wd)[BITS],
                                              const float2 (&xp)[MR][16],
                                              float2 (&acc)[MR]) {
  const float2 f = make_float2(code_as_float<BITS, 2 * J>(wd),
                               code_as_float<BITS, 2 * J + 1>(wd));
#pragma unroll
  for (int m = 0; m < MR; ++m) acc[m] = __ffma2_rn(f, xp[m][J], acc[m]);
}

template <int BITS, int MR, int... J>
__device__ __forceinline__ void unit_fma_impl(const uint32_t (&wd)[BITS],
                                              const float2 (&xp)[MR][16],
                                              float2 (&acc)[MR],
                                              std::integer_sequence<int, J...>) {
  (fma_code_pair<BITS, MR, J>(wd, xp, acc), ...);
}

// acc[m] += sum_i x''[m][i] * f_i over the 32 codes of one unit (two fp32
// lanes per accumulator; caller adds .x + .y).
template <int BITS, int MR>
__device__ __forceinline__ void unit_fma(const uint32_t (&wd)[BITS],
                                         const float2 (&xp)[MR][16],
                                         float2 (&acc)[MR]) {
  unit_fma_impl<BITS, MR>(wd, xp, acc, std::make_integer_sequence<int, 16>{});
}

// Load one unit (BITS words) from shared memory, using the widest aligned
// vector loads: a unit starts at a multiple of 4*BITS bytes.
template <int BITS>
__device__ __forceinline__ void load_unit(const uint32_t *p,
                                          uint32_t (&wd)[BITS]) {
  if constexpr (BITS % 4 == 0) {
#pragma unroll
    for (int i = 0; i < BITS / 4; ++i) {
      const uint4 v = reinterpret_cast<const uint4 *>(p)[i];
      wd[4 * i + 0] = v.x;
      wd[4 * i + 1] = v.y;
      wd[4 * i + 2] = v.z;
      wd[4 * i + 3] = v.w;
    }
  } else if constexpr (BITS % 2 == 0) {
#pragma unroll
    for (int i = 0; i < BITS / 2; ++i) {
      const uint2 v = reinterpret_cast<const uint2 *>(p)[i];
      wd[2 * i + 0] = v.x;
      wd[2 * i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < BITS; ++i) wd[i] = p[i];
  }
}

// Pre-scaled activations of one unit: xp[i] = v_i * 2^(149 - p_i - c),
// with c = max(22, E + 22) where max|v| < 2^E.  Returns 2^c and the plain
// sum of the 32 values (for the bias term).
template <int BITS>
__device__ __forceinline__ void prescale_unit(const float (&v)[32],
                                              float2 (&xp)[16], float &two_c,
                                              float &vsum) {
  float mx = 0.f;
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    mx = fmaxf(mx, fabsf(v[i]));
    s += v[i];
  }
  // biased exponent of max|v|: max|v| < 2^(eb - 126)
  const int eb = static_cast<int>((__float_as_uint(mx) >> 23) & 0xff);
  int c = eb - 126 + 22;
  c = c < 22 ? 22 : (c > 127 ? 127 : c);
  two_c = pow2i(c);
  vsum = s;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const float a = v[2 * j] * pow2i(149 - code_pos(BITS, 2 * j) - c);
    const float b = v[2 * j + 1] * pow2i(149 - code_pos(BITS, 2 * j + 1) - c);
    xp[j] = make_float2(a, b);
  }
}

}  // namespace qmvk
