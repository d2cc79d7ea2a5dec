// qmv_mma.cuh -- batched decode GEMV on the 5th-generation tensor cores.
//
// y[m, n] = sum_k x[m, k] * (scale[n, k/gs] * q[n, k] + bias[n, k/gs]) for a
// few activation rows (M <= 16) that share one read of the weights.  The
// product is a real contraction here, so it runs as
//     D[128 weight rows x 16] += W_hat[128 x 16 k] * X^T[16 k x 16]
// with tcgen05.mma (kind::f16, fp32 accumulation in tensor memory).
//
// One CTA per SM, three warp roles:
//   * producer (one thread): per stage, four 2-D tensor copies (TMA) into a
//     ring of shared-memory stages: 128 bytes of each of the tile's 128 packed
//     rows (128-byte swizzle), the matching window of each row's scales and
//     of its biases (32-byte swizzle), and the stage's slice of the M live x
//     rows; rows past N arrive as zeros;
//   * dequant warps (8; 16 for 2-bit codes): turn each stage into fp16
//     weights w_hat = scale * q + bias (a code made an exact fp16 value with
//     the 0x6400 magic, an exact fp16 correction, then one half2 FMA: a
//     single rounding, relative error below 2^-11) and write them straight
//     into tensor memory, where the MMA takes its A operand (row r of the
//     tile is tensor-memory lane r, so each warp writes the rows of its own
//     lane quarter); the chunk of x becomes the fp16 B operand in shared
//     memory (each x row scaled by its own power of two into fp16 range,
//     undone in the epilogue); at the end of a segment (the CTA's steps in
//     one tile) warps 0-3 read the accumulators and store y, or leave a
//     partial sum for the CTA that completes the tile;
//   * MMA warp: one thread issues the chunk's eight MMAs and commits them
//     to mbarriers; the warp also owns the tensor-memory allocation.
// Keeping A out of shared memory matters: in fp16 the weights are 4x (4-bit)
// to 8x (2-bit) their packed size, and writing them to shared memory and
// reading them back through the tensor core's descriptor path would cost
// more shared-memory bandwidth than the HBM stream delivers.
// The accumulators are double-buffered in tensor memory (two sets of
// kMmaNacc 16-column accumulators), so one segment's epilogue overlaps the
// next segment's MMAs.
//
// The order of k inside each group of 8 is permuted identically in W_hat
// and X^T (the nibble / byte pairing of the half2 unpack); a contraction
// does not depend on the order of k.
#pragma once

#include <cuda.h>

#include "qmv_device.cuh"

namespace qmvk {

struct MmaParams {
  const uint8_t *w;      // packed rows [N, K*bits/8]
  const uint16_t *s;     // scales bf16 [N, G]
  const uint16_t *b;     // biases bf16 [N, G]
  const uint16_t *x;     // bf16 [M, K]
  uint16_t *y;           // bf16 [M, N]
  int *err;              // OR 2 when a bounded wait gave up (null: none)
  int M, N, K, G;
  uint32_t row_bytes;    // K * bits / 8
  int ntiles;            // ceil(N / 128)
  int nstage;            // K / (codes per stage row)
  // Stream-K walk: the ntiles * nstage (tile, stage) steps, tile-major, are
  // cut into gridDim.x equal contiguous ranges, one per CTA (with as many
  // CTAs as tiles, every range is one whole tile).  A tile cut by
  // a range boundary leaves fp32 partial sums in `part` (two slots per CTA:
  // its first and its last segment, 16 x 128 floats each); the last CTA to
  // finish the tile (counted in cnt[tile], reset to 0 afterwards) adds the
  // parts in CTA order and stores y.
  long long nsteps;      // ntiles * nstage
  float *part;           // [gridDim.x][2][16][128]
  int *cnt;              // [ntiles], zero between launches
  int nst;               // stages in the shared-memory ring
  uint32_t stage_bytes;  // bytes of one stage (depends on M), 1024-aligned
  // dequant constants, passed in so that they live in registers for the
  // whole loop (an FMA or a 3-input logic op takes one immediate only)
  uint32_t k_magic;      // 0x64006400: fp16 1024 in each half
  uint32_t k_add[3];     // -1024 * 2^-SH in each half, SH = 2, 4, 6
};

constexpr int kMmaRows = 128;    // weight rows per tile (the MMA's M)
constexpr int kMmaKC = 128;      // K per chunk
constexpr int kMmaCols = 16;     // x rows per MMA (the MMA's N)
// fp16 A operands in flight in tensor memory (64 columns each, one per MMA
// chunk); the MMAs of a chunk complete well after they are issued, so the
// dequant warps run ahead
#ifndef QMV_MMA_NACC
#define QMV_MMA_NACC 4
#endif
// Independent accumulators per tile: the eight K = 16 MMAs of a chunk go
// round-robin to kMmaNacc accumulators (summed in the epilogue), so that
// consecutive MMAs do not wait on each other's result.
constexpr int kMmaNacc = QMV_MMA_NACC;
constexpr int kMmaAbufs = (512 - 2 * kMmaNacc * 16) / 64 < 7 ? (512 - 2 * kMmaNacc * 16) / 64 : 7;
constexpr uint32_t kMmaACols = kMmaKC / 2;             // 32-bit columns of one A
constexpr uint32_t kMmaDCol = kMmaAbufs * kMmaACols;   // first accumulator column
constexpr uint32_t kMmaTmemCols = 512;                 // allocation (power of two)

// Bytes of one fp16 B operand buffer (16 x 128).
constexpr uint32_t kMmaBBytes = kMmaCols * kMmaKC * 2;
// Core-matrix layout of B (K-major, no swizzle): element (row, k) of a
// buffer at (row / 8) * kMmaSBO + (k / 8) * kMmaLBO + (row % 8) * 16 + (k % 8) * 2.
constexpr uint32_t kMmaLBO = 128;                 // next 8 k
constexpr uint32_t kMmaSBO = (kMmaKC / 8) * 128;  // next 8 rows

// A stage holds 128 bytes of every row of the tile (a whole L2 line per
// row): 1024 / BITS codes, that is 1, 2 or 4 MMA chunks of 128 k.
template <int BITS>
__host__ __device__ constexpr int mma_stage_codes() { return 1024 / BITS; }
template <int BITS>
__host__ __device__ constexpr int mma_chunks_per_stage() { return 8 / BITS; }
// Scale / bias window of a row in a stage: 16 groups (32 bytes) from the
// stage's first group rounded down to a multiple of 8 (the copy's 16-byte
// start rule); that covers the stage's groups at every group size >= 32.
constexpr int kMmaWinGroups = 16;
// x arrives in slices of at most 256 codes (the copy's box limit).
template <int BITS>
__host__ __device__ constexpr int mma_x_slice() { return mma_stage_codes<BITS>() < 256 ? mma_stage_codes<BITS>() : 256; }

// Shared-memory plan (byte offsets from the dynamic shared base): the B
// operand buffers, barriers and small arrays first, then the ring of stages
// (1024-aligned: the 128-byte swizzle pattern repeats every 1024 bytes).
// A stage: the packed rows [128][128 B], the scale and bias windows
// [128][32 B], then the x slices [slice][M][slice codes] (bf16).
constexpr int kMmaMaxStages = 16;

template <int BITS>
struct MmaStage {
  static constexpr uint32_t s_off = kMmaRows * 128;
  static constexpr uint32_t b_off = s_off + kMmaRows * kMmaWinGroups * 2;
  static constexpr uint32_t x_off = b_off + kMmaRows * kMmaWinGroups * 2;
  static constexpr uint32_t x_row = mma_x_slice<BITS>() * 2;  // bytes per x row slice
  static constexpr uint32_t bytes(int M) {
    return (x_off + M * mma_stage_codes<BITS>() * 2 + 1023) / 1024 * 1024;
  }
  static constexpr uint32_t tx_bytes(int M) {  // bytes the copies of a stage deliver
    return x_off + M * mma_stage_codes<BITS>() * 2;
  }
};

struct MmaSmem {
  static constexpr uint32_t b_off = 0;
  static constexpr uint32_t bar_off = b_off + kMmaAbufs * kMmaBBytes;
  // wfull, wempty [kMmaMaxStages]; abfull, abempty [kMmaAbufs]; dfull, dempty [2]
  static constexpr uint32_t nbar = 2 * kMmaMaxStages + 2 * kMmaAbufs + 4;
  static constexpr uint32_t xinv_off = bar_off + nbar * 8;
  static constexpr uint32_t tmem_off = xinv_off + kMmaCols * 4;
  static constexpr uint32_t xmul_off = tmem_off + 16;
  static constexpr uint32_t flag_off = xmul_off + kMmaCols * 4;  // "this CTA ends the tile"
  static constexpr uint32_t w_off = (flag_off + 16 + 1023) / 1024 * 1024;
};

// ---------------------------------------------------------------------------
// tcgen05 helpers
// ---------------------------------------------------------------------------

// Shared-memory matrix descriptor: start address, leading (next 8 k) and
// stride (next 8 rows) byte offsets in 16-byte units, version 1, no swizzle.
__device__ __forceinline__ uint64_t mma_smem_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3fffu);
  d |= static_cast<uint64_t>((kMmaLBO >> 4) & 0x3fffu) << 16;
  d |= static_cast<uint64_t>((kMmaSBO >> 4) & 0x3fffu) << 32;
  d |= 1ull << 46;  // descriptor version
  return d;
}

// Instruction descriptor: fp32 accumulate, fp16 A and B, both K-major,
// N = 16, M = 128.
constexpr uint32_t kMmaIdesc = (1u << 4)                 // D format: f32
                             | ((kMmaCols >> 3) << 17)   // N / 8
                             | ((kMmaRows >> 4) << 24);  // M / 16

// D (tensor memory) += A (tensor memory, 128 lanes x 8 columns of fp16
// pairs) * B (shared memory, descriptor); accumulate = 0 overwrites D.
__device__ __forceinline__ void mma_f16_ta(uint32_t tmem_d, uint32_t tmem_a, uint64_t db,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n"
      "}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(db), "r"(kMmaIdesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u),
      "r"(0u)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}

// 32 lanes x 16 consecutive 32-bit columns of tensor memory.
__device__ __forceinline__ void tmem_ld16(uint32_t addr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
        "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
        "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(addr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 32 consecutive 32-bit columns of tensor memory (asynchronous:
// tmem_wait_st() waits for this thread's stores).
__device__ __forceinline__ void tmem_st32(uint32_t addr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n" ::"r"(
          addr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t addr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};\n" ::"r"(addr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t addr, const uint32_t *v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n" ::"r"(
          addr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}

__device__ __forceinline__ uint32_t lds16_mma(uint32_t a) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];\n" : "=h"(v) : "r"(a));
  return v;
}
// 2-D tensor copy global -> shared (box of the tensor map at (x, y)),
// completing its bytes on `bar`, with an L2 cache policy (the weights,
// scales and biases are read once per launch: evict-first, so they do not
// push the kernel's code and the activations out of L2).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;\n" : "=l"(pol));
  return pol;
}

// NG consecutive bf16 values (NG = 1, 2, 4, 8; aligned to NG) from shared
// memory, as 32-bit words (two values each, or one in the low half).
template <int NG>
__device__ __forceinline__ void lds_groups(uint32_t a, uint32_t (&v)[(NG + 1) / 2]) {
  if constexpr (NG == 1) {
    v[0] = lds16_mma(a);
  } else if constexpr (NG == 2) {
    asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v[0]) : "r"(a));
  } else if constexpr (NG == 4) {
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];\n" : "=r"(v[0]), "=r"(v[1]) : "r"(a));
  } else {
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                 : "r"(a));
  }
}

// Position in a ring of n slots: slot index and the parity of the lap.
struct RingPos {
  int idx = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void next(int n) {
    if (++idx == n) {
      idx = 0;
      phase ^= 1u;
    }
  }
};

// ---------------------------------------------------------------------------
// Dequant: one 32-bit word of codes -> fp16 w_hat, as half2 pairs, in the
// word's permuted k order (see the top of the file).
// ---------------------------------------------------------------------------
// h holds, in each fp16 half, 1024 + 2^SH * q exactly (a code q placed
// SH bits up in the mantissa under the 0x6400 exponent).  Recover q exactly,
// (h - 1024) or h * 2^-SH - 1024 * 2^-SH in one FMA, then
// w_hat = s * q + b with a single rounding.
__device__ __forceinline__ __half2 h2_bits(uint32_t v) {
  __half2 h;
  *reinterpret_cast<uint32_t *>(&h) = v;
  return h;
}
__device__ __forceinline__ uint32_t h2_u32(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }

template <int SH>
__device__ __forceinline__ uint32_t code_fma(uint32_t h, __half2 s2, __half2 b2,
                                             const uint32_t (&kadd)[3]) {
  __half2 q;
  if constexpr (SH == 0) {
    q = __hsub2(h2_bits(h), h2_bits(0x64006400u));
  } else {
    // h * 2^-SH + (-1024 * 2^-SH)
    constexpr uint32_t m = static_cast<uint32_t>(15 - SH) << 10;
    q = __hfma2(h2_bits(h), h2_bits(m | (m << 16)), h2_bits(kadd[SH / 2 - 1]));
  }
  return h2_u32(__hfma2(q, s2, b2));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// Codes of a word in k order 0..W-1 (W = 32 / BITS) become half2 values
// h[i] = (code a_i, code b_i); returns the number of half2 produced (W / 2).
//   8-bit: (0,2) (1,3)                       -> k order 0 2 1 3
//   4-bit: (0,4) (1,5) (2,6) (3,7)           -> k order 0 4 1 5 2 6 3 7
//   2-bit: (j, j+8) for j = 0..7             -> k order 0 8 1 9 ... 7 15
// Each code is masked in place (no shift per code; one shift by 8 serves
// the upper half of every 16-bit lane), so most of the work is on the
// fp16 pipe rather than the half-rate integer pipe.
template <int BITS>
__device__ __forceinline__ void dequant_word(uint32_t w, __half2 s2, __half2 b2, uint32_t kmagic,
                                             const uint32_t (&kadd)[3],
                                             uint32_t (&h)[16 / BITS]) {
  if constexpr (BITS == 8) {
    // bytes (0, 2) and (1, 3) under a 0x64 high byte
    h[0] = code_fma<0>(prmt(w, kmagic, 0x7250u), s2, b2, kadd);
    h[1] = code_fma<0>(prmt(w, kmagic, 0x7351u), s2, b2, kadd);
  } else if constexpr (BITS == 4) {
    const uint32_t v = w >> 8;
    h[0] = code_fma<0>((w & 0x000f000fu) | kmagic, s2, b2, kadd);
    h[1] = code_fma<4>((w & 0x00f000f0u) | kmagic, s2, b2, kadd);
    h[2] = code_fma<0>((v & 0x000f000fu) | kmagic, s2, b2, kadd);
    h[3] = code_fma<4>((v & 0x00f000f0u) | kmagic, s2, b2, kadd);
  } else {
    const uint32_t v = w >> 8;
    h[0] = code_fma<0>((w & 0x00030003u) | kmagic, s2, b2, kadd);
    h[1] = code_fma<2>((w & 0x000c000cu) | kmagic, s2, b2, kadd);
    h[2] = code_fma<4>((w & 0x00300030u) | kmagic, s2, b2, kadd);
    h[3] = code_fma<6>((w & 0x00c000c0u) | kmagic, s2, b2, kadd);
    h[4] = code_fma<0>((v & 0x00030003u) | kmagic, s2, b2, kadd);
    h[5] = code_fma<2>((v & 0x000c000cu) | kmagic, s2, b2, kadd);
    h[6] = code_fma<4>((v & 0x00300030u) | kmagic, s2, b2, kadd);
    h[7] = code_fma<6>((v & 0x00c000c0u) | kmagic, s2, b2, kadd);
  }
}

// The k offset, inside a span of codes, of element i (0..7) of the span's
// q-th core-matrix row of 8 fp16.  A span is the words that fill whole
// groups of 8: two 8-bit words (8 codes, one group), one 4-bit word (8
// codes, one group) or one 2-bit word (16 codes, two groups).  Element i is
// lane i % 2 of half2 number i / 2 of the unpack above.
__host__ __device__ constexpr int mma_k_of(int bits, int q, int i) {
  return bits == 8 ? (i / 4) * 4 + (i / 2) % 2 + 2 * (i % 2)
       : bits == 4 ? i / 2 + 4 * (i % 2)
                   : 4 * q + i / 2 + 8 * (i % 2);
}
template <int BITS>
__host__ __device__ constexpr int mma_span_codes() { return BITS == 2 ? 16 : 8; }

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(b), "f"(a));
  return r;  // a in the low half, b in the high half
}

// bf16 value in the low 16 bits -> (v, v) as an fp16 pair
__device__ __forceinline__ uint32_t bf16_to_half2_dup(uint32_t bits) {
  const float f = __uint_as_float(bits << 16);
  return pack_half2(f, f);
}


// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
// Dequant thread (r, qt): weight row r of the tile (tensor-memory lane r)
// and part qt of each stage row (NP parts of 128 / NP bytes, 1024 / (BITS *
// NP) codes).  A part lies inside one MMA chunk and fills 512 / (BITS * NP)
// of its 64 columns; the dequant warps number 4 * NP (a warp covers 32 rows
// of one part).
#ifndef QMV_MMA_PARTS
#define QMV_MMA_PARTS 2
#endif
template <int BITS>
__host__ __device__ constexpr int mma_parts() {
  return BITS == 2 ? 4 : QMV_MMA_PARTS;  // a 2-bit part must not cross a chunk
}
template <int BITS>
__host__ __device__ constexpr int mma_part_codes() { return 1024 / BITS / mma_parts<BITS>(); }
template <int BITS>
__host__ __device__ constexpr int mma_warps_per_chunk() { return 4 * (kMmaKC / mma_part_codes<BITS>()); }
template <int BITS>
__host__ __device__ constexpr int mma_threads() { return (4 * mma_parts<BITS>() + 2) * 32; }

// First step of CTA i's range, and the CTA whose range holds step v.
__device__ __forceinline__ long long mma_range_start(long long i, long long nsteps, int grid) {
  return i * nsteps / grid;
}
__device__ __forceinline__ int mma_range_of(long long v, long long nsteps, int grid) {
  return static_cast<int>(((v + 1) * grid - 1) / nsteps);
}

template <int BITS, int GS>
__global__ void __launch_bounds__(mma_threads<BITS>(), 1)
    qmv_mma_kernel(const __grid_constant__ CUtensorMap tm_w,
                   const __grid_constant__ CUtensorMap tm_s,
                   const __grid_constant__ CUtensorMap tm_b,
                   const __grid_constant__ CUtensorMap tm_x, const MmaParams p) {
  using ST = MmaStage<BITS>;
  constexpr int CPS = mma_chunks_per_stage<BITS>();   // MMA chunks per stage
  constexpr int SC = mma_stage_codes<BITS>();         // codes per stage row
  constexpr int NP = mma_parts<BITS>();               // parts per stage row
  constexpr int NAB = kMmaAbufs;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = smem_u32(smem);
  // the stage ring, 1024-aligned in the shared window (the launch reserves
  // 1 KB of slack for this)
  const uint32_t ring = (base + MmaSmem::w_off + 1023u) & ~1023u;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + MmaSmem::bar_off);
  uint64_t *wfull = bars, *wempty = bars + kMmaMaxStages;
  uint64_t *abfull = bars + 2 * kMmaMaxStages, *abempty = abfull + NAB;
  uint64_t *dfull = abempty + NAB, *dempty = dfull + 2;
  float *xinv = reinterpret_cast<float *>(smem + MmaSmem::xinv_off);
  float *xmul = reinterpret_cast<float *>(smem + MmaSmem::xmul_off);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + MmaSmem::tmem_off);
  constexpr int nw = 4 * NP;  // dequant warps: 0 .. nw-1
  const int nst = p.nst;
  const uint32_t sbytes = p.stage_bytes;
  grid_launch_dependents();

  // ---- set-up: barriers, tensor memory, x row ranges ----
  if (warp == nw) {
    if (lane < nst) {
      mbar_init(&wfull[lane], 1);  // the producer's expect_tx arrival
      mbar_init(&wempty[lane], nw);
    }
    if (lane < NAB) {
      mbar_init(&abfull[lane], mma_warps_per_chunk<BITS>());
      mbar_init(&abempty[lane], 1);  // tcgen05.commit
    }
    if (lane < 2) {
      mbar_init(&dfull[lane], 1);    // tcgen05.commit
      mbar_init(&dempty[lane], 4);   // the four epilogue warps
    }
    if (lane < kMmaCols) reinterpret_cast<int *>(xmul)[lane] = 0;  // max |x| bits
    fence_mbar_init();
  }
  if (warp == nw + 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kMmaTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  // the first global access of every thread follows (x, then the copies and
  // the stores): wait for the previous grid here, after the on-chip set-up
  grid_dependency_wait();
  __syncthreads();
  if (warp < nw) {
    // max |x| of each x row, over all K, by all dequant threads
    constexpr int nthr = nw * 32;
    for (int m = 0; m < p.M; ++m) {
      float mx = 0.f;
      const uint4 *row = reinterpret_cast<const uint4 *>(p.x + static_cast<size_t>(m) * p.K);
      for (int i = tid; i < p.K / 8; i += nthr) {
        const uint4 v = __ldg(row + i);
        const uint32_t ww[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          mx = fmaxf(mx, fabsf(__uint_as_float(ww[j] << 16)));
          mx = fmaxf(mx, fabsf(__uint_as_float(ww[j] & 0xffff0000u)));
        }
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) atomicMax(reinterpret_cast<int *>(xmul) + m, __float_as_int(mx));
    }
    // x rows M..15 of every B buffer are zeros, written once
    for (int i = tid; i < NAB * kMmaCols * (kMmaKC / 8); i += nthr) {
      const int buf = i / (kMmaCols * (kMmaKC / 8));
      const int rem = i % (kMmaCols * (kMmaKC / 8));
      const int row = rem / (kMmaKC / 8), kg = rem % (kMmaKC / 8);
      if (row >= p.M) {
        const uint32_t a = base + MmaSmem::b_off + buf * kMmaBBytes + (row / 8) * kMmaSBO +
                           kg * kMmaLBO + (row % 8) * 16;
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};\n" ::"r"(a), "r"(0u) : "memory");
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp < nw && tid < kMmaCols) {
    // x row m is scaled by 2^a with max|x| * 2^a in [2^13, 2^14): inside
    // fp16's range with room for the products' partial sums in fp32
    const float mx = __int_as_float(reinterpret_cast<int *>(xmul)[tid]);
    float inv = 1.0f, mul = 1.0f;
    if (tid < p.M && mx > 0.f) {
      const int eb = static_cast<int>((__float_as_uint(mx) >> 23) & 0xff);  // mx < 2^(eb-126)
      int a = 140 - eb;  // mx * 2^a < 2^14
      a = a < -126 ? -126 : (a > 126 ? 126 : a);
      mul = pow2i(a);
      inv = pow2i(-a);
    }
    xinv[tid] = inv;
    xmul[tid] = mul;
  }
  if (warp < nw) named_sync(1, nw * 32);  // dequant warps only (the multipliers)
  const uint32_t tmem_base = *tmem_slot;
  const long long v0 = mma_range_start(blockIdx.x, p.nsteps, gridDim.x);
  const long long v1 = mma_range_start(blockIdx.x + 1, p.nsteps, gridDim.x);

  if (warp == nw) {
    // ---------------- producer (one thread) ----------------
    // Per stage: the tile's 128 rows x 128 bytes of codes, 128 x 16 groups
    // of scales and of biases from group wg (a multiple of 8), and the x
    // slices; one expect_tx arrival announces all of their bytes.
    if (lane == 0) {
      RingPos sp;
      long long issued = 0;
      bool dead = false;
      constexpr int XS = mma_x_slice<BITS>();
      const uint32_t tx = ST::tx_bytes(p.M);
      const uint64_t pol_stream = l2_policy_evict_first();  // read once
      const uint64_t pol_keep = l2_policy_evict_last();     // x: read by every tile
      const uint32_t xstep = p.M * ST::x_row;
      int t = static_cast<int>(v0 / p.nstage), c = static_cast<int>(v0 % p.nstage);
      for (long long v = v0; v < v1; ++v, ++issued) {
        {
          const int r0 = t * kMmaRows;
          if (issued >= nst && !dead && !mbar_wait_sleep(&wempty[sp.idx], sp.phase ^ 1u))
            dead = true;
          const uint32_t dst = ring + sp.idx * sbytes;
          uint64_t *bar = &wfull[sp.idx];
          mbar_arrive_expect_tx(bar, tx);
          tma_load_2d(dst, &tm_w, c * 128, r0, bar, pol_stream);
          const int wg = (c * (SC / GS)) & ~7;
          tma_load_2d(dst + ST::s_off, &tm_s, wg, r0, bar, pol_stream);
          tma_load_2d(dst + ST::b_off, &tm_b, wg, r0, bar, pol_stream);
#pragma unroll
          for (int xs = 0; xs < SC / XS; ++xs)
            tma_load_2d(dst + ST::x_off + xs * xstep, &tm_x, c * SC + xs * XS, 0, bar,
                        pol_keep);
          sp.next(nst);
        }
        if (++c == p.nstage) {
          c = 0;
          ++t;
        }
      }
      // every copy issued must land before the CTA exits: wait (bounded)
      // for the last phase of each stage in use, the oldest first
      const int inuse = issued < nst ? static_cast<int>(issued) : nst;
      // once the ring has wrapped, the oldest stage in use is the next one
      // to issue, one lap back (phase parity flipped); before, stage 0
      RingPos q = sp;
      q.phase ^= 1u;
      if (issued < nst) q = RingPos();
      for (int i = 0; i < inuse; ++i) {
        if (!dead && !mbar_wait_sleep(&wfull[q.idx], q.phase)) dead = true;
        q.next(nst);
      }
      if (dead && p.err) atomicOr(p.err, 2);
    }
    __syncwarp();
  } else if (warp == nw + 1) {
    // ---------------- MMA warp ----------------
    RingPos ap;  // operand buffer position
    int sidx = 0;  // segments done (accumulator buffer position)
    bool dead = false;
    const uint64_t bdesc0 = mma_smem_desc(base + MmaSmem::b_off);
    int c = static_cast<int>(v0 % p.nstage);
    bool seg_start = true;
    uint32_t tmem_d = 0;
    int db = 0;
    for (long long v = v0; v < v1; ++v) {
      if (seg_start) {
        db = sidx & 1;
        const uint32_t dph = static_cast<uint32_t>((sidx >> 1) & 1);
        if (sidx >= 2 && !dead && !mbar_wait_sleep(&dempty[db], dph ^ 1u)) dead = true;
        tc_fence_after();
        tmem_d = tmem_base + kMmaDCol + db * (kMmaNacc * kMmaCols);
      }
      const bool seg_end = (c == p.nstage - 1) || (v == v1 - 1);
#pragma unroll 1
      for (int h = 0; h < CPS; ++h) {
        if (!dead && !mbar_wait_sleep(&abfull[ap.idx], ap.phase)) dead = true;
        tc_fence_after();
        if (lane == 0) {
          // descriptors advance by whole 16-byte units inside the start
          // address field (shared addresses stay below 2^18)
          const uint32_t a0 = tmem_base + ap.idx * kMmaACols;
          const uint64_t d0 = bdesc0 + static_cast<uint64_t>(ap.idx * (kMmaBBytes >> 4));
          if (seg_start && h == 0) {
#pragma unroll
            for (int j = 0; j < kMmaKC / 16; ++j)
              mma_f16_ta(tmem_d + (j % kMmaNacc) * kMmaCols, a0 + j * 8,
                         d0 + static_cast<uint64_t>(j * (2 * kMmaLBO >> 4)), j >= kMmaNacc ? 1u : 0u);
          } else {
#pragma unroll
            for (int j = 0; j < kMmaKC / 16; ++j)
              mma_f16_ta(tmem_d + (j % kMmaNacc) * kMmaCols, a0 + j * 8,
                         d0 + static_cast<uint64_t>(j * (2 * kMmaLBO >> 4)), 1u);
          }
          mma_commit(&abempty[ap.idx]);
          if (seg_end && h == CPS - 1) mma_commit(&dfull[db]);
        }
        __syncwarp();
        ap.next(NAB);
      }
      if (seg_end) ++sidx;
      seg_start = seg_end;
      if (++c == p.nstage) c = 0;
    }
    if (dead && p.err && lane == 0) atomicOr(p.err, 2);
  } else {
    // ---------------- dequant warps ----------------
    const int r = tid % kMmaRows;
    const int qt = tid / kMmaRows;                   // part of the stage row
    constexpr int QW = 32 / NP;                      // words per part
    constexpr int QC = mma_part_codes<BITS>();       // codes per part
    constexpr int NV = QC / 2;                       // tensor-memory columns written
    constexpr int SPAN = mma_span_codes<BITS>();     // codes per span
    constexpr int WPS = SPAN * BITS / 32;            // words per span
    constexpr int GPS = SPAN / 8;                    // core rows per span
    constexpr int NSP = QW / WPS;                    // spans per part
    constexpr int NG = QC >= GS ? QC / GS : 1;       // groups in a part
    const int cc = (qt * QC) / kMmaKC;               // MMA chunk within the stage
    // per-thread offsets, fixed for the whole launch
    uint32_t woff[QW / 4];  // the part's 16-byte chunks in the swizzled row
#pragma unroll
    for (int i = 0; i < QW / 4; ++i)
      woff[i] = r * 128 + (((((QW / 4) * qt + i) ^ (r & 7)) & 7) << 4);
    const int gpart = (qt * QC) / GS;  // the part's first group, from the stage's
    const uint32_t wrow = r * 32;
    const uint32_t wswz = static_cast<uint32_t>((r >> 2) & 1);
    const uint32_t ta0 = tmem_base + (static_cast<uint32_t>(32 * (warp % 4)) << 16) +
                         static_cast<uint32_t>((qt * QC) % kMmaKC) / 2;
    // x writers: a chunk's B operand is 16 * M units (x row m, core row kg
    // of 8 k), dealt over the TW threads that write the chunk's A; unit u
    // goes to writer u % TW (rows >= M stay zero)
    constexpr int TW = kMmaRows * (kMmaKC / QC);
    constexpr int UPT = (kMmaCols * (kMmaKC / 8) + TW - 1) / TW;  // units per writer, at most
    const int xw = r + kMmaRows * (qt % (kMmaKC / QC));          // writer index
    const int nunits = p.M * (kMmaKC / 8);
    uint32_t xsrc[UPT], xdst[UPT], xq[UPT];
    float xm[UPT];
#pragma unroll
    for (int ui = 0; ui < UPT; ++ui) {
      const int u = xw + ui * TW;
      const int m = u < nunits ? u / (kMmaKC / 8) : 0, kg = u % (kMmaKC / 8);
      constexpr int XS = mma_x_slice<BITS>();
      const int xk = cc * kMmaKC + (kg / GPS) * SPAN;  // the span's first code in the stage
      xsrc[ui] = ST::x_off + ((xk / XS) * p.M + m) * ST::x_row + (xk % XS) * 2;
      xdst[ui] = MmaSmem::b_off + (m / 8) * kMmaSBO + kg * kMmaLBO + (m % 8) * 16;
      xq[ui] = kg % GPS;
      xm[ui] = xmul[m];
    }
    const uint32_t kmagic = p.k_magic;
    const uint32_t kadd[3] = {p.k_add[0], p.k_add[1], p.k_add[2]};
    RingPos sp, ap;
    // this thread's first operand buffer: chunk cc of the first stage
    for (int i = 0; i < cc; ++i) ap.next(NAB);
    long long kc = cc;  // MMA chunk count of this thread's chunk
    bool dead = false;
    const bool x_warp = (xw & ~31) < nunits;  // this warp writes B units
    // What a stage leaves in registers: the part's words, its groups'
    // scale / bias pairs and the x spans behind this thread's B units.
    struct Regs {
      uint32_t wd[QW];
      __half2 s2[NG], b2[NG];
      uint4 xv[UPT][SPAN / 8];
    };
    // Wait for stage c of the ring, read this thread's share of it, then
    // hand the stage back to the producer.
    auto load = [&](Regs &R, int c) {
      if (!dead && !mbar_wait(&wfull[sp.idx], sp.phase)) dead = true;
      const uint32_t stg = ring + sp.idx * sbytes;
#pragma unroll
      for (int i = 0; i < QW / 4; ++i)
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n"
                     : "=r"(R.wd[4 * i]), "=r"(R.wd[4 * i + 1]), "=r"(R.wd[4 * i + 2]),
                       "=r"(R.wd[4 * i + 3])
                     : "r"(stg + woff[i]));
      // NG groups from window index gh (a multiple of NG, so one aligned
      // load); 32-byte swizzle: 16-byte chunk j of row r at j ^ ((r / 4) % 2)
      const int gh = ((c * (SC / GS)) & 7) + gpart;
      const uint32_t wo = wrow + ((((2 * gh) >> 4) ^ wswz) << 4) + ((2 * gh) & 15);
      uint32_t sv[(NG + 1) / 2], bv[(NG + 1) / 2];
      lds_groups<NG>(stg + ST::s_off + wo, sv);
      lds_groups<NG>(stg + ST::b_off + wo, bv);
#pragma unroll
      for (int ui = 0; ui < UPT; ++ui) {
        if (xw + ui * TW < nunits) {
#pragma unroll
          for (int i = 0; i < SPAN / 8; ++i)
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n"
                         : "=r"(R.xv[ui][i].x), "=r"(R.xv[ui][i].y), "=r"(R.xv[ui][i].z),
                           "=r"(R.xv[ui][i].w)
                         : "r"(stg + xsrc[ui] + 16 * i));
        }
      }
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        R.s2[g] = h2_bits(bf16_to_half2_dup((sv[g / 2] >> (16 * (g % 2))) & 0xffffu));
        R.b2[g] = h2_bits(bf16_to_half2_dup((bv[g / 2] >> (16 * (g % 2))) & 0xffffu));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&wempty[sp.idx]);
      sp.next(nst);
    };
    // Stage (t, c) from registers R: fp16 weights into tensor memory, the x
    // units into the B buffer; the next stage is read into N while the
    // stores drain, then the chunk is handed to the MMA warp.
    // the walk: step v of the CTA's range is stage c of tile t; the current
    // segment (the range's steps inside one tile) began at stage cseg0
    long long v = v0;
    int t = static_cast<int>(v0 / p.nstage), c = static_cast<int>(v0 % p.nstage);
    int cseg0 = c, sidx = 0;
    int *tile_flag = reinterpret_cast<int *>(smem + MmaSmem::flag_off);
    auto step = [&](Regs &R, Regs &N) {
      // the operand buffer must be free: its previous MMAs have completed
      if (kc >= NAB && !dead && !mbar_wait(&abempty[ap.idx], ap.phase ^ 1u)) dead = true;
      tc_fence_after();
      uint32_t av[NV];
#pragma unroll
      for (int s = 0; s < NSP; ++s) {
        const int g = (QC >= GS) ? (s * SPAN) / GS : 0;  // compile time
#pragma unroll
        for (int wi = 0; wi < WPS; ++wi) {
          uint32_t hw[16 / BITS];
          dequant_word<BITS>(R.wd[s * WPS + wi], R.s2[g], R.b2[g], kmagic, kadd, hw);
#pragma unroll
          for (int j = 0; j < 16 / BITS; ++j) av[(s * WPS + wi) * (16 / BITS) + j] = hw[j];
        }
      }
      const uint32_t ta = ta0 + ap.idx * kMmaACols;
#ifndef QMV_MMA_ST
#define QMV_MMA_ST 32
#endif
      constexpr int STC = QMV_MMA_ST < NV ? QMV_MMA_ST : NV;  // columns per store
      if constexpr (STC == 8) {
#pragma unroll
        for (int i = 0; i < NV / 8; ++i) tmem_st8(ta + 8 * i, &av[8 * i]);
      } else if constexpr (STC == 16) {
#pragma unroll
        for (int i = 0; i < NV / 16; ++i)
          tmem_st16(ta + 16 * i, *reinterpret_cast<const uint32_t(*)[16]>(&av[16 * i]));
      } else {
#pragma unroll
        for (int i = 0; i < NV / 32; ++i)
          tmem_st32(ta + 32 * i, *reinterpret_cast<const uint32_t(*)[32]>(&av[32 * i]));
      }
      const uint32_t bbuf = base + ap.idx * kMmaBBytes;
#pragma unroll
      for (int ui = 0; ui < UPT; ++ui) {
        if (xw + ui * TW < nunits) {
          float xs[SPAN];
#pragma unroll
          for (int i = 0; i < SPAN / 8; ++i) {
            const uint32_t qq[4] = {R.xv[ui][i].x, R.xv[ui][i].y, R.xv[ui][i].z, R.xv[ui][i].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              xs[8 * i + 2 * j] = __uint_as_float(qq[j] << 16) * xm[ui];
              xs[8 * i + 2 * j + 1] = __uint_as_float(qq[j] & 0xffff0000u) * xm[ui];
            }
          }
          uint32_t hv[4];
          if (GPS == 1 || xq[ui] == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              hv[i] = pack_half2(xs[mma_k_of(BITS, 0, 2 * i)], xs[mma_k_of(BITS, 0, 2 * i + 1)]);
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              hv[i] = pack_half2(xs[mma_k_of(BITS, 1, 2 * i)], xs[mma_k_of(BITS, 1, 2 * i + 1)]);
          }
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};\n" ::"r"(bbuf + xdst[ui]),
                       "r"(hv[0]), "r"(hv[1]), "r"(hv[2]), "r"(hv[3])
                       : "memory");
        }
      }
      // the next stage of this CTA's walk
      const int tc = t;
      const bool seg_end = (c == p.nstage - 1) || (v == v1 - 1);
      const bool whole_tile = seg_end && cseg0 == 0 && c == p.nstage - 1;
      ++v;
      if (++c == p.nstage) {
        c = 0;
        ++t;
      }
      if (seg_end) cseg0 = c;
      if (v < v1) load(N, c);
      tmem_wait_st();
      // make the tensor-memory stores, and the B units' generic-proxy
      // shared stores, visible to the MMA
      if (x_warp) asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&abfull[ap.idx]);
      for (int i = 0; i < CPS; ++i) ap.next(NAB);
      kc += CPS;
      // ---- epilogue of the segment: warps 0..3 read the accumulator ----
      if (seg_end) {
        if (warp < 4) {
          const int db = sidx & 1;
          const uint32_t dph = static_cast<uint32_t>((sidx >> 1) & 1);
          if (!dead && !mbar_wait(&dfull[db], dph)) dead = true;
          tc_fence_after();
          float d[16];
          const uint32_t dcol = tmem_base + (static_cast<uint32_t>(32 * warp) << 16) + kMmaDCol +
                                db * (kMmaNacc * kMmaCols);
          tmem_ld16(dcol, d);
#pragma unroll
          for (int a = 1; a < kMmaNacc; ++a) {
            float e[16];
            tmem_ld16(dcol + a * kMmaCols, e);
#pragma unroll
            for (int m = 0; m < 16; ++m) d[m] += e[m];
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&dempty[db]);
          const int rt = 32 * warp + lane;  // row in the tile
          const int row = tc * kMmaRows + rt;
          if (whole_tile) {
            if (row < p.N) {
#pragma unroll
              for (int m = 0; m < kMmaCols; ++m)
                if (m < p.M) p.y[static_cast<size_t>(m) * p.N + row] = f32_to_bf16(d[m] * xinv[m]);
            }
          } else {
            // a part of tile tc: leave it in this CTA's slot (0 for the
            // range's first segment, 1 for its last), count it, and if it
            // is the tile's last part to arrive, add all parts in CTA order
            const long long ts = static_cast<long long>(tc) * p.nstage;
            const int first = mma_range_of(ts, p.nsteps, gridDim.x);
            const int last = mma_range_of(ts + p.nstage - 1, p.nsteps, gridDim.x);
            float *mine = p.part + (static_cast<size_t>(blockIdx.x) * 2 + (v0 >= ts ? 0 : 1)) *
                                       (kMmaCols * kMmaRows);
#pragma unroll
            for (int m = 0; m < kMmaCols; ++m)
              if (m < p.M) mine[m * kMmaRows + rt] = d[m];
            __threadfence();
            named_sync(2, 128);
            if (warp == 0 && lane == 0)
              *tile_flag = atomicAdd(&p.cnt[tc], 1) == last - first ? 1 : 0;
            named_sync(2, 128);
            if (*tile_flag) {
              __threadfence();
              float acc[16];
#pragma unroll
              for (int m = 0; m < kMmaCols; ++m) acc[m] = 0.f;
              for (int j = first; j <= last; ++j) {
                if (j == static_cast<int>(blockIdx.x)) {
#pragma unroll
                  for (int m = 0; m < kMmaCols; ++m) acc[m] += d[m];
                } else {
                  const long long sj = mma_range_start(j, p.nsteps, gridDim.x);
                  const float *pj = p.part + (static_cast<size_t>(j) * 2 + (sj >= ts ? 0 : 1)) *
                                                 (kMmaCols * kMmaRows);
#pragma unroll
                  for (int m = 0; m < kMmaCols; ++m)
                    if (m < p.M) acc[m] += __ldcg(pj + m * kMmaRows + rt);
                }
              }
              if (row < p.N) {
#pragma unroll
                for (int m = 0; m < kMmaCols; ++m)
                  if (m < p.M)
                    p.y[static_cast<size_t>(m) * p.N + row] = f32_to_bf16(acc[m] * xinv[m]);
              }
              if (warp == 0 && lane == 0) p.cnt[tc] = 0;  // ready for the next launch
            }
          }
        }
        ++sidx;
      }
    };
    Regs A, B;
    if (v < v1) load(A, c);
    while (v < v1) {
      step(A, B);
      if (v >= v1) break;
      step(B, A);
    }
    if (dead && p.err && lane == 0) atomicOr(p.err, 2);
  }
  // ---- tear-down: the tensor memory goes back once every reader is done ----
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == nw + 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem_base),
                 "r"(kMmaTmemCols)
                 : "memory");
}

}  // namespace qmvk
