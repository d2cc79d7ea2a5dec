// qmv_decode.cuh -- the decode GEMV kernel: one activation row per weight
// matrix, on the CUDA cores.  It serves y = x @ dequant(W).T, the dual
// gate/up product and the SiLU-gated down projection for 2- and 4-bit codes
// and rows of a multiple of 2048 codes (the decode shapes).
//
// Each CTA (one per SM) owns a contiguous block of output rows and streams
// their packed weights, scales and biases through a ring of shared-memory
// slots with 1-D bulk copies.  Two warp roles:
//   * consumer warps (at most 16; a thread holds at most 96 registers):
//     a thread owns one 64-code "span" of the rows -- the same columns of
//     every row it touches -- and keeps the span's activations in registers
//     as three 8-bit digits of an exact 22-bit fixed-point value per code,
//     met by the codes spread into byte lanes in dp4a (exact integer dot
//     products).  For every slot it computes its span of the slot's rows (two
//     rows interleaved), applies each
//     group's scale and bias, reduces the row partials over the warp with
//     shuffles and leaves one partial per (row, warp of the row) in shared
//     memory;
//   * producer warp: issues the slot copies and, once the consumers have
//     released a slot, adds the partials of each of its rows in a fixed
//     order, adds the residual, rounds once to bf16 and stores.
// The activation digits are prepared once per CTA: every consumer thread
// turns 16 activations into digits and writes them to shared memory, then
// every thread loads the digits of its own span (one span's digits serve all
// the row phases that touch it).
//
// Scales and biases enter as sc * sum(q * x) + bias * sum(x) per group, the
// algebra of the pages' qdot ("mlx/include/mlx/backend/metal/kernels/
// quantized.h", MLX 0.30.1); the integer digits replace that kernel's
// pre-scaled activations.
#pragma once

#include "qmv_device.cuh"

namespace qmvk {

constexpr int kSpan = 64;          // codes per consumer thread and row
constexpr int kDecodeMaxWarps = 16;

constexpr int kDecodeRps = 2;      // rows per row phase and slot (interleaved)
// Words of a span's shared-memory record: the activation digits [3][16] and
// three constants, padded to 16 bytes.
constexpr int kSpanRec = 52;

struct DecodeParams {
  const uint8_t *w[2];    // packed rows of matrix 0 / 1 (gate / up)
  const uint16_t *s[2];   // scales bf16 [N, G]
  const uint16_t *b[2];   // biases bf16 [N, G]
  uint16_t *y[2];         // outputs bf16 [N]
  const uint16_t *x;      // bf16 [K]; SiLU mode: gate
  const uint16_t *up;     // SiLU mode: up [K]
  const uint16_t *resid;  // SiLU mode: x_resid [N] or null
  int *err;               // OR 2 when a bounded wait gave up (null: none)
  long long total_rows;   // nmat * N
  int N, K, G;            // rows per matrix, codes per row, groups per row
  int WPR;                // consumer warps per row: K / 2048
  int PH;                 // row phases: consumer warps / WPR
  int SR;                 // rows per slot: PH * kDecodeRps
  int nslot;              // slots in the ring
  uint32_t row_bytes;     // K * bits / 8
  uint32_t slot_w;        // bytes of a slot's packed rows (SR * row_bytes)
  uint32_t slot_s;        // bytes of a slot's scales (SR * 2G); biases follow
  uint32_t slot_bytes;    // slot_w + 2 * slot_s, rounded up to 128
  uint32_t part_off;      // smem offset: partials [nslot][2][SR][WPR] floats
  uint32_t dig_off;       // smem offset: span records [K / 64][kSpanRec]
  uint32_t x_off;         // smem offset: the activations (x; SiLU: gate, up)
  uint32_t bar_off;       // smem offset: full[nslot], empty[nslot]
};

// The CTA's rows, slot by slot: rows [T*c/G, T*(c+1)/G) of the nmat*N rows
// (G CTAs), cut into slots of at most SR rows that stay inside one matrix.
struct SlotWalk {
  long long i, end;
  int N, SR;
  __device__ __forceinline__ void init(const DecodeParams &p) {
    i = p.total_rows * blockIdx.x / gridDim.x;
    end = p.total_rows * (blockIdx.x + 1) / gridDim.x;
    N = p.N;
    SR = p.SR;
  }
  // the next slot: rows [row, row + n) of matrix m
  __device__ __forceinline__ bool next(int &m, int &row, int &n) {
    if (i >= end) return false;
    m = i >= N ? 1 : 0;
    const long long me = static_cast<long long>(m + 1) * N;
    long long e = i + SR;
    if (e > end) e = end;
    if (e > me) e = me;
    row = static_cast<int>(i - static_cast<long long>(m) * N);
    n = static_cast<int>(e - i);
    i = e;
    return true;
  }
};

// ---------------------------------------------------------------------------
// Codes in byte lanes.  The span's 64 codes are 2*BITS words; spread
// register r (0..15) holds four of them, one per byte, for dp4a:
//   8-bit: word r;  4-bit: the even (r even) or odd nibbles of word r/2;
//   2-bit: the 2-bit fields at shift 2*(r%4) of each byte of word r/4.
// Lane j of register r is code spread_code(BITS, r, j) of the span, and the
// registers 0..7 hold exactly the codes 0..31.
// ---------------------------------------------------------------------------
template <int BITS>
__device__ __forceinline__ uint32_t span_spread(const uint32_t *wd, int r) {
  if constexpr (BITS == 8) {
    return wd[r];
  } else if constexpr (BITS == 4) {
    const uint32_t w = wd[r >> 1];
    return ((r & 1) ? (w >> 4) : w) & 0x0F0F0F0Fu;
  } else {
    return (wd[r >> 2] >> (2 * (r & 3))) & 0x03030303u;
  }
}

// ---------------------------------------------------------------------------
// Activation digits.  A span's activations v (x, or silu(gate) * up in fp32)
// become X = rint(v * 2^s) with one power of two per span chosen so that
// |X| < 2^22 (exact for every element within 2^14 of the span's largest
// magnitude; smaller ones are rounded to the span's grid).  X's three low
// bytes are its digits: X = d0 + 2^8 d1 + 2^16 d2 with d0, d1 unsigned and
// d2 signed.  A span's record in shared memory: digits [3][16] in the spread
// layout (word d*16 + r holds digit d of the four codes of spread register
// r), then 2^-s, the plain sum of the activations of each group part (one
// part, or two for group size 32), and a pad word.
//
// Work item i covers activations [16 i, 16 i + 16): the quarter i % 4 of
// span i / 4, whose four items are consecutive lanes of one warp.
// ---------------------------------------------------------------------------
template <int BITS, int GS, bool SILU>
__device__ __forceinline__ void prepare_digits(const DecodeParams &p, uint32_t xs,
                                               uint32_t rec_base, int ctid, int nthreads) {
  const int items = p.K / 16;
  const unsigned full = 0xffffffffu;
  for (int it = ctid; it < items; it += nthreads) {
    const int q = it & 3;
    const uint32_t off = static_cast<uint32_t>(it) * 32;  // bytes into x
    float v[16];
    {
      const uint4 a = lds128(xs + off), b = lds128(xs + off + 16);
      const uint32_t xw[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        v[2 * h] = __uint_as_float(xw[h] << 16);
        v[2 * h + 1] = __uint_as_float(xw[h] & 0xffff0000u);
      }
    }
    if constexpr (SILU) {
      // silu(g) = g / (1 + e^-g) with the fast exponential and division
      // (relative error near 2^-21); held in fp32, never rounded to bf16
      const uint32_t us = xs + 2u * static_cast<uint32_t>(p.K);
      const uint4 a = lds128(us + off), b = lds128(us + off + 16);
      const uint32_t uw[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        const float u0 = __uint_as_float(uw[h] << 16);
        const float u1 = __uint_as_float(uw[h] & 0xffff0000u);
        const float g0 = v[2 * h], g1 = v[2 * h + 1];
        v[2 * h] = __fdividef(g0, 1.0f + __expf(-g0)) * u0;
        v[2 * h + 1] = __fdividef(g1, 1.0f + __expf(-g1)) * u1;
      }
    }
    float mx = 0.f, sum = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      mx = fmaxf(mx, fabsf(v[j]));
      sum += v[j];
    }
    // span maximum over its four quarters; sums per group part
    mx = fmaxf(mx, __shfl_xor_sync(full, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(full, mx, 2));
    sum += __shfl_xor_sync(full, sum, 1);
    if constexpr (GS != 32) sum += __shfl_xor_sync(full, sum, 2);
    const int eb = static_cast<int>((__float_as_uint(mx) >> 23) & 0xff);
    const uint32_t rec = rec_base + static_cast<uint32_t>(it >> 2) * (kSpanRec * 4);
    float cst;  // the record's scale-back constant
    {
      int sh = 148 - eb;  // max|v| < 2^(eb - 126), so |v| * 2^sh < 2^22
      sh = sh < -126 ? -126 : (sh > 126 ? 126 : sh);
      const float sc = pow2i(sh);
      cst = pow2i(-sh);
      int X[16];
#pragma unroll
      for (int j = 0; j < 16; ++j)
        X[j] = __float_as_int(fmaf(v[j], sc, kDigitBiasF)) - kDigitBias;
      // spread registers 4q .. 4q+3 take their codes from this quarter
      uint32_t dg[3][4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int c0 = spread_code(BITS, r, 0), c1 = spread_code(BITS, r, 1);
        const int c2 = spread_code(BITS, r, 2), c3 = spread_code(BITS, r, 3);
        const int a = X[c0], b = X[c1], c = X[c2], d = X[c3];
        const uint32_t ab = __byte_perm(a, b, 0x5140);   // a0 b0 a1 b1
        const uint32_t cd = __byte_perm(c, d, 0x5140);   // c0 d0 c1 d1
        dg[0][r] = __byte_perm(ab, cd, 0x5410);          // a0 b0 c0 d0
        dg[1][r] = __byte_perm(ab, cd, 0x7632);          // a1 b1 c1 d1
        const uint32_t ab2 = __byte_perm(a, b, 0x0062);  // a2 b2
        const uint32_t cd2 = __byte_perm(c, d, 0x0062);  // c2 d2
        dg[2][r] = __byte_perm(ab2, cd2, 0x5410);        // a2 b2 c2 d2
      }
#pragma unroll
      for (int d = 0; d < 3; ++d)
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};\n" ::"r"(rec + (d * 16 + 4 * q) * 4),
                     "r"(dg[d][0]), "r"(dg[d][1]), "r"(dg[d][2]), "r"(dg[d][3])
                     : "memory");
    }
    constexpr int kc = kSpanRec - 4;  // the constants' first word
    if (q == 0) {
      asm volatile("st.shared.v2.f32 [%0], {%1, %2};\n" ::"r"(rec + kc * 4), "f"(cst), "f"(sum)
                   : "memory");
      if constexpr (GS != 32)
        asm volatile("st.shared.f32 [%0], %1;\n" ::"r"(rec + (kc + 2) * 4), "f"(0.f) : "memory");
    } else if (GS == 32 && q == 2) {
      asm volatile("st.shared.f32 [%0], %1;\n" ::"r"(rec + (kc + 2) * 4), "f"(sum) : "memory");
    }
  }
}

// The codes of quarter-local spread register r (0..3) are the quarter's
// activations spread_code(BITS, r, j) for j = 0..3: with 16 codes per
// quarter, register 4q + r of the span holds codes 16q + spread_code(BITS,
// r, j).  (spread_code(BITS, 4q + r, j) = 16q + spread_code(BITS, r, j) for
// every width.)
static_assert(spread_code(4, 5, 2) == 16 + spread_code(4, 1, 2), "spread layout");
static_assert(spread_code(2, 13, 3) == 48 + spread_code(2, 1, 3), "spread layout");
static_assert(spread_code(8, 10, 1) == 32 + spread_code(8, 2, 1), "spread layout");

// ---------------------------------------------------------------------------
// NR rows (1 or 2) of one span: for each row, sum over the span's codes of
// x * w_hat, as (sum_h sc_h * sum(q * X)_h) * 2^-s + sum_h bias_h * sum(v)_h.
// The rows' dot products are interleaved (independent dp4a chains).
// aw[j]: the span's packed words of row j; as[j]: the row's scales (its
// biases follow slot_s bytes later).
// ---------------------------------------------------------------------------
template <int BITS, int GS, int NR>
__device__ __forceinline__ void span_rows(const uint32_t (&aw)[NR], const uint32_t (&as)[NR],
                                          uint32_t slot_s, const uint32_t (&dig)[3][16],
                                          float back, const float (&vsum)[2], float (&out)[NR]) {
  constexpr int NW = 2 * BITS;             // packed words of the span
  constexpr int NGP = GS == 32 ? 2 : 1;    // group parts of the span
  uint32_t wd[NR][NW];
#pragma unroll
  for (int j = 0; j < NR; ++j)
#pragma unroll
    for (int i = 0; i < NW / 4; ++i) {
      const uint4 v = lds128(aw[j] + 16 * i);
      wd[j][4 * i] = v.x;
      wd[j][4 * i + 1] = v.y;
      wd[j][4 * i + 2] = v.z;
      wd[j][4 * i + 3] = v.w;
    }
  uint32_t sw[NR], bw[NR];
#pragma unroll
  for (int j = 0; j < NR; ++j) {
    if constexpr (NGP == 2) {
      sw[j] = lds32(as[j]);  // two consecutive groups
      bw[j] = lds32(as[j] + slot_s);
    } else {
      sw[j] = lds16(as[j]);
      bw[j] = lds16(as[j] + slot_s);
    }
  }
  int acc[NR][NGP][3];
#pragma unroll
  for (int j = 0; j < NR; ++j)
#pragma unroll
    for (int h = 0; h < NGP; ++h) acc[j][h][0] = acc[j][h][1] = acc[j][h][2] = kDigitBias;
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const int h = NGP == 2 ? r / 8 : 0;
#pragma unroll
    for (int j = 0; j < NR; ++j) {
      const uint32_t c = span_spread<BITS>(wd[j], r);
      acc[j][h][0] = dp4a_uu(dig[0][r], c, acc[j][h][0]);
      acc[j][h][1] = dp4a_uu(dig[1][r], c, acc[j][h][1]);
      acc[j][h][2] = dp4a_su(dig[2][r], c, acc[j][h][2]);
    }
  }
#pragma unroll
  for (int j = 0; j < NR; ++j) {
    float sr = 0.f, bs = 0.f;
#pragma unroll
    for (int h = 0; h < NGP; ++h) {
      // each digit sum read as a float is 1.5 * 2^23 + sum exactly
      const float t0 = __int_as_float(acc[j][h][0]) - kDigitBiasF;
      const float t1 = fmaf(__int_as_float(acc[j][h][1]), 256.f, -256.f * kDigitBiasF);
      const float t2 = fmaf(__int_as_float(acc[j][h][2]), 65536.f, -65536.f * kDigitBiasF);
      const float r = t0 + t1 + t2;
      const float sc = __uint_as_float(h == 0 ? (sw[j] << 16) : (sw[j] & 0xffff0000u));
      const float bi = __uint_as_float(h == 0 ? (bw[j] << 16) : (bw[j] & 0xffff0000u));
      sr = fmaf(sc, r, sr);
      bs = fmaf(bi, vsum[h], bs);
    }
    out[j] = fmaf(sr, back, bs);
  }
}

__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(pol));
  return pol;
}

// One bulk copy global -> shared in chunks of at most 16 KB, completing on
// `bar`, with an L2 cache policy.  Addresses 16-byte aligned, bytes a
// multiple of 16.
__device__ __forceinline__ void bulk_copy_pol(uint32_t dst, const uint8_t *src,
                                              uint32_t bytes, uint64_t *bar,
                                              uint64_t pol) {
  constexpr uint32_t kChunk = 16384;
  for (uint32_t o = 0; o < bytes; o += kChunk) {
    const uint32_t n = bytes - o < kChunk ? bytes - o : kChunk;
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1], %2, [%3], %4;\n" ::"r"(dst + o),
        "l"(src + o), "r"(n), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
  }
}

// ---------------------------------------------------------------------------
// Producer warp: fills the ring, and drains it slot by slot: after the
// consumers released a slot it refills the slot with the next rows, then
// finishes the released rows (partials of the row's warps added in order,
// residual, one rounding, store).
// ---------------------------------------------------------------------------
template <bool SILU>
__device__ __forceinline__ void decode_producer(const DecodeParams &p, uint32_t sbase,
                                                uint64_t *full, uint64_t *empty,
                                                const float *part, int lane) {
  const uint64_t pol = l2_evict_first();
  const uint32_t sg_bytes = 2u * p.G;
  auto issue = [&](int slot, int m, int row, int n) {
    if (lane != 0) return;
    const uint32_t dst = sbase + static_cast<uint32_t>(slot) * p.slot_bytes;
    uint64_t *bar = &full[slot];
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(n) * (p.row_bytes + 2 * sg_bytes));
    bulk_copy_pol(dst, p.w[m] + static_cast<size_t>(row) * p.row_bytes,
                  static_cast<uint32_t>(n) * p.row_bytes, bar, pol);
    bulk_copy_pol(dst + p.slot_w,
                  reinterpret_cast<const uint8_t *>(p.s[m]) + static_cast<size_t>(row) * sg_bytes,
                  static_cast<uint32_t>(n) * sg_bytes, bar, pol);
    bulk_copy_pol(dst + p.slot_w + p.slot_s,
                  reinterpret_cast<const uint8_t *>(p.b[m]) + static_cast<size_t>(row) * sg_bytes,
                  static_cast<uint32_t>(n) * sg_bytes, bar, pol);
  };
  SlotWalk fill, drain;
  fill.init(p);
  drain = fill;
  int nfill = 0;
  int m, row, n;
  // Nothing is read before the previous grid (which may write any of the
  // inputs) has finished; then the ring fills at once.
  grid_dependency_wait();
  while (nfill < p.nslot && fill.next(m, row, n)) issue(nfill++, m, row, n);
  int slot = 0;
  uint32_t par = 0;
  bool dead = false;
  while (drain.next(m, row, n)) {
    if (!dead && !mbar_wait_sleep(&empty[slot], par)) dead = true;
    {
      int m2, row2, n2;
      if (fill.next(m2, row2, n2)) {
        issue(slot, m2, row2, n2);
        ++nfill;
      }
    }
    const float *pp = part + (static_cast<size_t>(slot) * 2 + par) * p.SR * p.WPR;
    if (lane < n) {
      float acc = 0.f;
      for (int w = 0; w < p.WPR; ++w) acc += pp[lane * p.WPR + w];
      const int r = row + lane;
      if constexpr (SILU) {
        if (p.resid) acc += bf16_to_f32(p.resid[r]);
      }
      p.y[m][r] = f32_to_bf16(acc);
    }
    __syncwarp();
    if (++slot == p.nslot) {
      slot = 0;
      par ^= 1u;
    }
  }
  if (dead && p.err && lane == 0) atomicOr(p.err, 2);
  // every copy must have landed before the CTA exits (normally the
  // consumers saw all of them already): the last use of each used slot
  for (int i = lane; i < p.nslot && i < nfill; i += 32) {
    const int last = (nfill - 1 - i) / p.nslot;
    mbar_wait_sleep(&full[i], static_cast<uint32_t>(last & 1));
  }
}

// A consumer thread's span activations in registers, loaded from its record.
template <int BITS>
struct SpanActs {
  uint32_t dig[3][16];
  __device__ __forceinline__ void load(uint32_t rec) {
#pragma unroll
    for (int i = 0; i < 12; ++i) {
      const uint4 v = lds128(rec + 16 * i);
      dig[i / 4][4 * (i % 4)] = v.x;
      dig[i / 4][4 * (i % 4) + 1] = v.y;
      dig[i / 4][4 * (i % 4) + 2] = v.z;
      dig[i / 4][4 * (i % 4) + 3] = v.w;
    }
  }
};
// ---------------------------------------------------------------------------
// The kernel.  Threads: NW consumer warps (NW = WPR * PH) then the producer
// warp.
// ---------------------------------------------------------------------------
template <int BITS, int GS, bool SILU>
__global__ void __launch_bounds__((kDecodeMaxWarps + 1) * 32, 1)
    qmv_decode_kernel(const DecodeParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x;
  const int NWc = p.WPR * p.PH;  // consumer warps
  const int Tc = NWc * 32;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + p.bar_off);
  uint64_t *empty = full + p.nslot;
  float *part = reinterpret_cast<float *>(smem + p.part_off);
  const uint32_t sbase = smem_u32(smem);
  grid_launch_dependents();

  if (tid >= Tc) {
    const int lane = tid & 31;
    for (int i = lane; i < p.nslot; i += 32) {
      mbar_init(&full[i], 1);      // the producer's expect-tx arrival
      mbar_init(&empty[i], NWc);   // one arrival per consumer warp
    }
    fence_mbar_init();
    __syncwarp();
    named_arrive(1, blockDim.x);
    decode_producer<SILU>(p, sbase, full, empty, part, lane);
    return;
  }

  // ---- consumers: this thread's span and row phase ----
  const int warp = tid >> 5, lane = tid & 31;
  const int ph = warp / p.WPR, wr = warp - ph * p.WPR;
  const int t = wr * 32 + lane;  // span index
  const uint32_t rec_base = sbase + p.dig_off;
  // the barriers are used after named barrier 1, which the producer passes
  // once it has initialised them
  named_sync(1, blockDim.x);
  bool dead = false;
  {
    // the activations (x; SiLU: gate then up) into shared memory, 16 bytes
    // per load, once the previous grid (which may write them) has finished
    grid_dependency_wait();
    const int nx = (SILU ? 2 : 1) * p.K / 8;
    const uint32_t xs = sbase + p.x_off;
    for (int i = tid; i < nx; i += Tc) {
      const uint4 v = i < p.K / 8 ? __ldg(reinterpret_cast<const uint4 *>(p.x) + i)
                                  : __ldg(reinterpret_cast<const uint4 *>(p.up) + (i - p.K / 8));
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};\n" ::"r"(xs + 16u * i), "r"(v.x),
                   "r"(v.y), "r"(v.z), "r"(v.w)
                   : "memory");
    }
    named_sync(2, Tc);
  }
  prepare_digits<BITS, GS, SILU>(p, sbase + p.x_off, rec_base, tid, Tc);
  named_sync(2, Tc);
  constexpr int RW = kSpanRec;
  SpanActs<BITS> sa;  // digits [3][16]
  float back, vsum[2];
  {
    const uint32_t rec = rec_base + static_cast<uint32_t>(t) * (RW * 4);
    sa.load(rec);
    const uint4 c = lds128(rec + (RW - 4) * 4);
    back = __uint_as_float(c.x);
    vsum[0] = __uint_as_float(c.y);
    vsum[1] = __uint_as_float(c.z);
  }

  const uint32_t sg_bytes = 2u * p.G;
  const uint32_t span_w = static_cast<uint32_t>(t) * (8 * BITS);   // bytes into a row
  const uint32_t span_s = 2u * static_cast<uint32_t>((t * kSpan) / GS);
  SlotWalk walk;
  walk.init(p);
  int slot = 0;
  uint32_t par = 0;
  int m, row, n;
  while (walk.next(m, row, n)) {
    if (!dead && !mbar_wait_sleep(&full[slot], par)) dead = true;
    const uint32_t base = sbase + static_cast<uint32_t>(slot) * p.slot_bytes;
    const uint32_t wb = base + span_w, sb = base + p.slot_w + span_s;
    const int l0 = ph, l1 = ph + p.PH;
    float pr[2] = {0.f, 0.f};
    const uint32_t(&dig)[3][16] = sa.dig;
    if (l1 < n) {  // warp-uniform
      const uint32_t aw[2] = {wb + static_cast<uint32_t>(l0) * p.row_bytes,
                              wb + static_cast<uint32_t>(l1) * p.row_bytes};
      const uint32_t as[2] = {sb + static_cast<uint32_t>(l0) * sg_bytes,
                              sb + static_cast<uint32_t>(l1) * sg_bytes};
      span_rows<BITS, GS, 2>(aw, as, p.slot_s, dig, back, vsum, pr);
    } else if (l0 < n) {
      const uint32_t aw[1] = {wb + static_cast<uint32_t>(l0) * p.row_bytes};
      const uint32_t as[1] = {sb + static_cast<uint32_t>(l0) * sg_bytes};
      float o[1];
      span_rows<BITS, GS, 1>(aw, as, p.slot_s, dig, back, vsum, o);
      pr[0] = o[0];
    }
    transpose_reduce<2>(pr, lane);
    float *pp = part + (static_cast<size_t>(slot) * 2 + par) * p.SR * p.WPR;
    if ((lane & 15) == 0) {
      const int lr = ph + p.PH * (lane >> 4);
      if (lr < n) pp[lr * p.WPR + wr] = pr[0];
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
    if (++slot == p.nslot) {
      slot = 0;
      par ^= 1u;
    }
  }
  if (dead && p.err && lane == 0) atomicOr(p.err, 2);
}

}  // namespace qmvk
