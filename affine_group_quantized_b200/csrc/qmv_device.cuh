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

// Bounded wait that lets the waiting thread sleep: each try_wait may
// suspend the thread for up to 10 us, or until the phase completes.  The
// bound (2^16 rounds, well under a second) only ends a broken launch.
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < (1u << 16); ++i) {
    uint32_t ok;
    asm volatile(
        "{\n"
        ".reg .pred p;\n"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        "selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(10000u)
        : "memory");
    if (ok) return true;
  }
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

// Programmatic dependent launch: a kernel launched right behind another on
// the same stream may be scheduled before that one has finished; it waits
// here, before its first global memory access, until the previous grid has
// completed and its writes are visible (a no-op for an ordinary launch).
// launch_dependents lets the next grid get scheduled as SMs free up.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
}
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

// Named barrier `id` over `nthreads` threads (a multiple of 32): wait for
// all of them, or only signal arrival without waiting.
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void named_arrive(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.arrive %0, %1;\n" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------
// Shared-memory helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];\n" : "=h"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}

// ---------------------------------------------------------------------------
// Warp reductions
// ---------------------------------------------------------------------------

// c ? a : b on values, kept a register select (a select between two array
// elements may otherwise become an indexed load from local memory).
__device__ __forceinline__ float select_f32(bool c, float a, float b) {
  float r;
  asm("{\n.reg .pred q;\nsetp.ne.u32 q, %3, 0;\nselp.f32 %0, %1, %2, q;\n}\n"
      : "=f"(r)
      : "f"(a), "f"(b), "r"(static_cast<uint32_t>(c)));
  return r;
}

// Transposed butterfly over the 32 lanes of a warp: NV partial sums per lane
// in; afterwards lane l holds the full sum of value l / (32 / NV) in vals[0].
template <int NV>
__device__ __forceinline__ void transpose_reduce(float (&vals)[NV], int lane) {
  static_assert(NV >= 1 && NV <= 32 && (NV & (NV - 1)) == 0, "NV");
  const unsigned full = 0xffffffffu;
#pragma unroll
  for (int off = 16, n = NV; off >= 1; off >>= 1) {
    if (n > 1) {
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < n / 2; ++i) {
        const float lo = vals[i], hi = vals[i + n / 2];
        const float send = select_f32(upper, lo, hi);
        const float keep = select_f32(upper, hi, lo);
        vals[i] = keep + __shfl_xor_sync(full, send, off);
      }
      n >>= 1;
    } else {
      vals[0] += __shfl_xor_sync(full, vals[0], off);
    }
  }
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

// Two rows of one unit at a time: the codes of both rows are decoded and fed
// to fp32 FMAs against the same pre-scaled activations.  Each row keeps four
// accumulators, so the eight FMA chains of a row pair are independent and the
// decode instructions interleave with them.
template <int BITS, int MR, int J>
__device__ __forceinline__ void fma_pair_2rows(const uint32_t (&w0)[BITS],
                                               const uint32_t (&w1)[BITS],
                                               const float2 (&xp)[MR][16],
                                               float2 (&a0)[MR][2],
                                               float2 (&a1)[MR][2]) {
  // scalar FMAs: packed fp32x2 FMAs would need the two decoded codes moved
  // into a register pair first, which costs more than it saves
  const float f0x = code_as_float<BITS, 2 * J>(w0);
  const float f0y = code_as_float<BITS, 2 * J + 1>(w0);
  const float f1x = code_as_float<BITS, 2 * J>(w1);
  const float f1y = code_as_float<BITS, 2 * J + 1>(w1);
#pragma unroll
  for (int m = 0; m < MR; ++m) {
    a0[m][J & 1].x = fmaf(f0x, xp[m][J].x, a0[m][J & 1].x);
    a0[m][J & 1].y = fmaf(f0y, xp[m][J].y, a0[m][J & 1].y);
    a1[m][J & 1].x = fmaf(f1x, xp[m][J].x, a1[m][J & 1].x);
    a1[m][J & 1].y = fmaf(f1y, xp[m][J].y, a1[m][J & 1].y);
  }
}

template <int BITS, int MR, int... J>
__device__ __forceinline__ void unit_fma_2rows_impl(
    const uint32_t (&w0)[BITS], const uint32_t (&w1)[BITS],
    const float2 (&xp)[MR][16], float2 (&a0)[MR][2], float2 (&a1)[MR][2],
    std::integer_sequence<int, J...>) {
  (fma_pair_2rows<BITS, MR, J>(w0, w1, xp, a0, a1), ...);
}

// a{0,1}[m][*] += x''[m][i] * f_i over the 32 codes of one unit of rows 0/1.
// The caller sums the four fp32 lanes of each row.
template <int BITS, int MR>
__device__ __forceinline__ void unit_fma_2rows(const uint32_t (&w0)[BITS],
                                               const uint32_t (&w1)[BITS],
                                               const float2 (&xp)[MR][16],
                                               float2 (&a0)[MR][2],
                                               float2 (&a1)[MR][2]) {
  unit_fma_2rows_impl<BITS, MR>(w0, w1, xp, a0, a1,
                                std::make_integer_sequence<int, 16>{});
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


// ---------------------------------------------------------------------------
// Integer path for 2-, 4- and 8-bit codes.
//
// The 32 codes of a unit are spread into eight 32-bit registers holding four
// codes each, one per byte (8-bit: the words themselves; 4-bit: the even and
// the odd nibbles of each word, masked; 2-bit: the four 2-bit lanes of each
// byte, shifted and masked).  The activations of the unit are turned into
// 22-bit fixed point relative to the unit's largest magnitude,
// X_i = rint(x_i * 2^s) with |X_i| <= 2^22, and the three low bytes of X_i's
// two's-complement form are its digits: X = sext(b2) * 2^16 + b1 * 2^8 + b0
// with b0, b1 unsigned.  Every digit register holds one digit of the four
// activations that meet the four codes of one code register, so dp4a (four
// 8-bit products added to a 32-bit integer) computes sum_i q_i * b_i exactly.
// X_i equals x_i * 2^s exactly whenever |x_i| is within 2^14 of the unit's
// largest |x| (a bf16 carries 8 significant bits); smaller elements are
// rounded to the unit's grid, an error below 2^-23 of the unit's largest |x|.
// Each digit sum starts from 0x4B400000, the bit pattern of 1.5 * 2^23: as
// long as |sum| < 2^22 the 32-bit result read as a float is 1.5 * 2^23 + sum
// exactly, so no integer-to-float conversion is needed; the same constant
// rounds x * 2^s to an integer with one fused multiply-add.
// ---------------------------------------------------------------------------

template <int BITS>
constexpr bool kIntPath = BITS == 2 || BITS == 4 || BITS == 8;

constexpr int kDigitBias = 0x4B400000;        // bits of 12582912.0f
constexpr float kDigitBiasF = 12582912.0f;

// (register, byte lane) of code i of a unit in the spread layout
__host__ __device__ constexpr int spread_reg(int bits, int i) {
  return bits == 8 ? i / 4
       : bits == 4 ? 2 * (i / 8) + (i % 8) % 2
                   : 4 * (i / 16) + (i % 16) % 4;
}
__host__ __device__ constexpr int spread_lane(int bits, int i) {
  return bits == 8 ? i % 4 : bits == 4 ? (i % 8) / 2 : (i % 16) / 4;
}
// code index held in byte lane `lane` of spread register r
__host__ __device__ constexpr int spread_code(int bits, int r, int lane) {
  return bits == 8 ? 4 * r + lane
       : bits == 4 ? 8 * (r / 2) + (r % 2) + 2 * lane
                   : 16 * (r / 4) + (r % 4) + 4 * lane;
}

// Spread register R (0..7) of a unit: four codes, one per byte.
template <int BITS, int R>
__device__ __forceinline__ uint32_t spread_codes(const uint32_t (&wd)[BITS]) {
  if constexpr (BITS == 8) {
    return wd[R];
  } else if constexpr (BITS == 4) {
    const uint32_t w = wd[R / 2];
    return (R % 2 == 0 ? w : (w >> 4)) & 0x0F0F0F0Fu;
  } else {
    const uint32_t w = wd[R / 4];
    return (w >> (2 * (R % 4))) & 0x03030303u;
  }
}

// dp4a with unsigned (low digits) or signed (top digit) activation bytes;
// the code bytes are unsigned.
__device__ __forceinline__ int dp4a_uu(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.u32.u32 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp4a_su(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp4a.s32.u32 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Digits of the unit's activations in the spread layout, the scale back to
// activation units (2^-s) and the plain activation sum times 2^s.
template <int BITS>
__device__ __forceinline__ void digits_unit(const float (&v)[32],
                                            uint32_t (&dig)[3][8], float &inv,
                                            float &vs) {
  float mx = 0.f, sum = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    mx = fmaxf(mx, fabsf(v[i]));
    sum += v[i];
  }
  const int eb = static_cast<int>((__float_as_uint(mx) >> 23) & 0xff);
  int s = 148 - eb;  // max|v| < 2^(eb-126), so |v| * 2^s < 2^22
  s = s < -126 ? -126 : (s > 126 ? 126 : s);
  const float sc = pow2i(s);
  inv = pow2i(-s);
  vs = sum * sc;
  int X[32];
#pragma unroll
  for (int i = 0; i < 32; ++i)
    X[i] = __float_as_int(fmaf(v[i], sc, kDigitBiasF)) - kDigitBias;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int a = X[spread_code(BITS, r, 0)], b = X[spread_code(BITS, r, 1)];
    const int c = X[spread_code(BITS, r, 2)], d = X[spread_code(BITS, r, 3)];
    const uint32_t ab = __byte_perm(a, b, 0x5140);  // a0 b0 a1 b1
    const uint32_t cd = __byte_perm(c, d, 0x5140);  // c0 d0 c1 d1
    dig[0][r] = __byte_perm(ab, cd, 0x5410);        // a0 b0 c0 d0
    dig[1][r] = __byte_perm(ab, cd, 0x7632);        // a1 b1 c1 d1
    const uint32_t ab2 = __byte_perm(a, b, 0x0062); // a2 b2
    const uint32_t cd2 = __byte_perm(c, d, 0x0062); // c2 d2
    dig[2][r] = __byte_perm(ab2, cd2, 0x5410);      // a2 b2 c2 d2
  }
}

template <int BITS, int MR, int R>
__device__ __forceinline__ void dp_reg_2rows(const uint32_t (&w0)[BITS],
                                             const uint32_t (&w1)[BITS],
                                             const uint32_t (&dig)[MR][3][8],
                                             int (&a0)[MR][3], int (&a1)[MR][3]) {
  const uint32_t b0 = spread_codes<BITS, R>(w0);
  const uint32_t b1 = spread_codes<BITS, R>(w1);
#pragma unroll
  for (int m = 0; m < MR; ++m) {
    a0[m][0] = dp4a_uu(dig[m][0][R], b0, a0[m][0]);
    a0[m][1] = dp4a_uu(dig[m][1][R], b0, a0[m][1]);
    a0[m][2] = dp4a_su(dig[m][2][R], b0, a0[m][2]);
    a1[m][0] = dp4a_uu(dig[m][0][R], b1, a1[m][0]);
    a1[m][1] = dp4a_uu(dig[m][1][R], b1, a1[m][1]);
    a1[m][2] = dp4a_su(dig[m][2][R], b1, a1[m][2]);
  }
}

template <int BITS, int MR, int... R>
__device__ __forceinline__ void unit_dp_2rows_impl(
    const uint32_t (&w0)[BITS], const uint32_t (&w1)[BITS],
    const uint32_t (&dig)[MR][3][8], int (&a0)[MR][3], int (&a1)[MR][3],
    std::integer_sequence<int, R...>) {
  (dp_reg_2rows<BITS, MR, R>(w0, w1, dig, a0, a1), ...);
}

// sum_i q_i * X_i of one unit for two rows, as floats (exact up to the last
// two additions).
template <int BITS, int MR>
__device__ __forceinline__ void unit_dp_2rows(const uint32_t (&w0)[BITS],
                                              const uint32_t (&w1)[BITS],
                                              const uint32_t (&dig)[MR][3][8],
                                              float (&r0)[MR], float (&r1)[MR]) {
  int a0[MR][3], a1[MR][3];
#pragma unroll
  for (int m = 0; m < MR; ++m)
#pragma unroll
    for (int l = 0; l < 3; ++l) a0[m][l] = a1[m][l] = kDigitBias;
  unit_dp_2rows_impl<BITS, MR>(w0, w1, dig, a0, a1,
                               std::make_integer_sequence<int, 8>{});
#pragma unroll
  for (int m = 0; m < MR; ++m) {
    r0[m] = fmaf(__int_as_float(a0[m][2]) - kDigitBiasF, 65536.f,
                 fmaf(__int_as_float(a0[m][1]) - kDigitBiasF, 256.f,
                      __int_as_float(a0[m][0]) - kDigitBiasF));
    r1[m] = fmaf(__int_as_float(a1[m][2]) - kDigitBiasF, 65536.f,
                 fmaf(__int_as_float(a1[m][1]) - kDigitBiasF, 256.f,
                      __int_as_float(a1[m][0]) - kDigitBiasF));
  }
}

}  // namespace qmvk
