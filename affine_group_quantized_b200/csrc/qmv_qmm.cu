// qmv_qmm.cu -- y = x @ dequant(W).T for many activation rows (the pages'
// qmm_t: "mlx/include/mlx/backend/metal/kernels/quantized.h", qmm_t_impl
// and affine_qmm_t, MLX 0.30.1) on the 5th-generation tensor cores.
//
//   D[128 weight rows x MC] += W_hat[128 x 16 k] * X^T[16 k x MC]
//
// with tcgen05.mma kind::f16, both operands bf16, fp32 accumulation in
// tensor memory.  MC (16, 32, 64 or 128) activation rows form a column block;
// a launch covers (weight tile, column block) tiles, column blocks inner,
// so a weight tile's later blocks read it again from L2.
//
// W_hat is the dequantized weight itself: bf16(scale * q + bias) with one
// rounding (one bf16 fused multiply-add on an exact code), the value the
// library's dequantize writes.  The x rows are the B operand straight from
// memory: the tensor-copy engine (TMA) writes each 128-k chunk of MC rows
// as two 128-byte-swizzled boxes, the layout the MMA's shared-memory
// descriptor reads.  Nothing scales or converts x.
//
// One CTA per SM, the roles of the few-row kernel (qmv_mma.cuh):
//   * producer (one thread): per stage, the tile's 128 rows x 128 bytes of
//     codes and their scale / bias windows into a ring of stages, and per
//     128-k chunk the x boxes into a second ring of x slots;
//   * dequant warps: codes -> bf16 W_hat in natural k order, written to
//     tensor memory (row r of the tile is lane r); at the end of a segment
//     (a CTA's steps in one tile) they also read the accumulator and store
//     y, or leave a partial sum for the CTA that completes the tile;
//   * MMA warp: one thread issues each chunk's eight K = 16 MMAs and
//     commits them to the barriers that free the A buffer and the x slot.
// The (tile, stage) steps are cut into equal contiguous ranges, one per CTA
// (stream-K); a tile cut by a range boundary is added up from fp32 partial
// sums in CTA order, so results do not depend on timing.  Without scratch
// the ranges are whole tiles.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "qmv.h"
#include "qmv_mma.cuh"
#include "qmv_qmm.h"

namespace qmvk {

template <int MC>
struct QmmShape {
  // MMA-issuing warps: a thread issues an MMA about every 25 ns whatever its
  // size, while the tensor core takes one of N <= 64 in about 10-18 ns, so
  // narrow blocks spread their chunks over two issuers (chunk j of a segment
  // goes to issuer j % 2), each with its own accumulator; the epilogue adds
  // them in issuer order
  static constexpr int kIssuers = MC >= 128 ? 1 : 2;
  static constexpr int kNacc = 1;                         // accumulators per issuer
  static constexpr int kDCols = 2 * kIssuers * MC;        // double-buffered
  static constexpr int kAbufs = (512 - kDCols) / 64 < 7 ? (512 - kDCols) / 64 : 7;
  static constexpr uint32_t kDCol = kAbufs * 64;  // first accumulator column
  // accumulator of issuer i in buffer db
  static constexpr uint32_t dcol(int db, int i) { return kDCol + (db * kIssuers + i) * MC; }
  static constexpr uint32_t kXBytes = MC * 256;   // one x chunk: MC rows x 128 k bf16
  // fp32 D, bf16 A and B, both K-major, N = MC, M = 128
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                     (static_cast<uint32_t>(MC >> 3) << 17) |
                                     (static_cast<uint32_t>(kMmaRows >> 4) << 24);
  static_assert(kAbufs >= 4, "tensor memory plan");
};

constexpr int kQmmMaxX = 8;  // x slots, at most
constexpr int kQmmMaxAbufs = 7;

// A stage holds SB = 128 bytes of each of the tile's 128 rows (one box,
// 128-byte swizzle), then the rows' scale and bias windows: 16 groups (32
// bytes) from the stage's first group rounded down to a multiple of 8 (the
// copy's 16-byte start rule), which covers the stage's groups at every group
// size for SB * 8 / BITS <= 512 codes.
template <int BITS>
struct QmmStage {
  static constexpr int SB = 128;                                // bytes of a row per stage
  static constexpr int SC = SB * 8 / BITS;                      // codes of a row per stage
  static constexpr int CPS = SC / kMmaKC;                       // MMA chunks per stage
  static constexpr int NBOX = SB / 128;
  static constexpr uint32_t s_off = kMmaRows * SB;
  static constexpr uint32_t b_off = s_off + kMmaRows * kMmaWinGroups * 2;
  static constexpr uint32_t bytes = b_off + kMmaRows * kMmaWinGroups * 2;
  static_assert(SC <= 512 && bytes % 1024 == 0, "stage plan");
};

// Dequant thread (r, qt): weight row r of the tile (tensor-memory lane r)
// and part qt of each stage row: a quarter of the row's SB bytes, so 16
// dequant warps (a warp covers 32 rows of one part); a part lies inside one
// MMA chunk.
constexpr int kQmmParts = 4;
template <int BITS>
__host__ __device__ constexpr int qmm_part_codes() { return QmmStage<BITS>::SC / kQmmParts; }
template <int BITS>
__host__ __device__ constexpr int qmm_warps_per_chunk() { return 4 * (kMmaKC / qmm_part_codes<BITS>()); }
template <int MC>
__host__ __device__ constexpr int qmm_threads() { return (4 * kQmmParts + 1 + QmmShape<MC>::kIssuers) * 32; }

struct QmmSmem {
  // wfull, wempty [kMmaMaxStages]; xfull, xempty [kQmmMaxX];
  // abfull, abempty [kQmmMaxAbufs]; dfull, dempty [2]
  static constexpr uint32_t nbar = 2 * kMmaMaxStages + 2 * kQmmMaxX + 2 * kQmmMaxAbufs + 4;
  static constexpr uint32_t tmem_off = nbar * 8;
  static constexpr uint32_t flag_off = tmem_off + 16;
  static constexpr uint32_t ring_off = 1024;  // then x slots, then weight stages
  static_assert(flag_off + 16 <= ring_off, "shared-memory plan");
};

struct QmmParams {
  uint16_t *y;        // bf16 [M, N]
  int *err;           // OR 2 when a bounded wait gave up
  int M, N;
  int nmb;            // column blocks: ceil(M / MC)
  int nstage;         // K / (codes per stage row)
  long long nsteps;   // tiles * nstage
  long long gran;     // steps per schedule unit: 1 (stream-K) or nstage
  float *part;        // [gridDim.x][2][MC][128] partial sums (split tiles)
  int *cnt;           // [tiles], zero between launches
  int nst;            // weight stages in the ring
  int nxs;            // x slots in the ring
};

// First step of CTA i's range, and the CTA whose range holds step v
// (ranges are whole schedule units of `gran` steps).
__device__ __forceinline__ long long qmm_start(long long i, const QmmParams &p) {
  return (i * (p.nsteps / p.gran) / gridDim.x) * p.gran;
}
__device__ __forceinline__ int qmm_owner(long long v, const QmmParams &p) {
  const long long u = v / p.gran, nu = p.nsteps / p.gran;
  return static_cast<int>(((u + 1) * gridDim.x - 1) / nu);
}

// Shared-memory descriptor of a K-major operand in 128-byte-swizzled rows
// (8-row groups 1024 bytes apart), version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3fffu);
  d |= static_cast<uint64_t>(1u) << 16;             // leading offset (unused when swizzled)
  d |= static_cast<uint64_t>(1024u >> 4) << 32;     // next 8 rows
  d |= 1ull << 46;                                  // descriptor version
  d |= 2ull << 61;                                  // 128-byte swizzle
  return d;
}

template <int MC>
__device__ __forceinline__ void umma_bf16_ta(uint32_t tmem_d, uint32_t tmem_a, uint64_t db,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n"
      "}\n" ::"r"(tmem_d),
      "r"(tmem_a), "l"(db), "r"(QmmShape<MC>::kIdesc), "r"(accumulate), "r"(0u), "r"(0u),
      "r"(0u), "r"(0u)
      : "memory");
}

// The eight K = 16 MMAs of one 128-k chunk, all accumulating, from one asm
// block with their operands formed inside it: A at tensor-memory columns
// a0 + 8j; B's descriptor start field (16-byte units; shared addresses stay
// below 2^18, so the low word never carries) at box j / 4 of the chunk
// (MC * 128 bytes apart) and 32 bytes (16 k) per j inside the swizzled row;
// D round-robin over the accumulators (MC columns apart).  Few instructions
// per MMA matter: the issuing thread shares its scheduler with dequant warps.
template <int MC>
__device__ __forceinline__ void umma_chunk_acc(uint32_t d0, uint32_t a0, uint64_t b0) {
  constexpr int NA = QmmShape<MC>::kNacc;
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      ".reg .b32 bl, bh, t;\n"
      ".reg .b32 a1, a2, a3, a4, a5, a6, a7;\n"
      ".reg .b32 d1, d2, d3;\n"
      ".reg .b64 b1, b2, b3, b4, b5, b6, b7;\n"
      "setp.ne.b32 p, 1, 0;\n"
      "mov.b64 {bl, bh}, %2;\n"
      "add.u32 a1, %1, 8;\n add.u32 a2, %1, 16;\n add.u32 a3, %1, 24;\n add.u32 a4, %1, 32;\n"
      "add.u32 a5, %1, 40;\n add.u32 a6, %1, 48;\n add.u32 a7, %1, 56;\n"
      "add.u32 t, bl, 2;\n mov.b64 b1, {t, bh};\n"
      "add.u32 t, bl, 4;\n mov.b64 b2, {t, bh};\n"
      "add.u32 t, bl, 6;\n mov.b64 b3, {t, bh};\n"
      "add.u32 t, bl, %4;\n mov.b64 b4, {t, bh};\n"
      "add.u32 t, bl, %5;\n mov.b64 b5, {t, bh};\n"
      "add.u32 t, bl, %6;\n mov.b64 b6, {t, bh};\n"
      "add.u32 t, bl, %7;\n mov.b64 b7, {t, bh};\n"
      "add.u32 d1, %0, %8;\n add.u32 d2, %0, %9;\n add.u32 d3, %0, %10;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [d1], [a1], b1, %3, p;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [d2], [a2], b2, %3, p;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [d3], [a3], b3, %3, p;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [a4], b4, %3, p;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [d1], [a5], b5, %3, p;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [d2], [a6], b6, %3, p;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [d3], [a7], b7, %3, p;\n"
      "}\n" ::"r"(d0),
      "r"(a0), "l"(b0), "r"(QmmShape<MC>::kIdesc), "n"(MC * 8), "n"(MC * 8 + 2),
      "n"(MC * 8 + 4), "n"(MC * 8 + 6), "n"((1 % NA) * MC), "n"((2 % NA) * MC),
      "n"((3 % NA) * MC)
      : "memory");
}

__device__ __forceinline__ uint32_t bf2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;\n" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// One 32-bit word of codes (k order: the low bits first) -> bf16 pairs
// (w_hat[k], w_hat[k+1]) for consecutive k.  A code becomes an exact bf16
// number first: its bits under the exponent of 128 give 128 + 2^i q (the
// code i bits up in the mantissa, kept below the exponent field's lowest
// bit), and one pair FMA with exact constants gives q in each half; then
// w_hat = bf16(s * q + b) in one more FMA (a single rounding).  8-bit codes
// have more bits than the bf16 mantissa: they go through binary32
// (2^23 + q, minus 2^23) and an exact conversion of the integer pair.
template <int BITS>
__device__ __forceinline__ void unpack_word_bf16(uint32_t w, uint32_t s2, uint32_t b2,
                                                 uint32_t (&h)[16 / BITS]) {
  constexpr uint32_t kMagic = 0x43004300u;  // bf16 128 in each half
  if constexpr (BITS == 4) {
    // pair p is byte p: low nibble (code 2p) in the low half, high nibble
    // (code 2p+1) one bit down in the high half, i.e. 128 + 8 q
    const uint32_t w1 = w >> 1;
#pragma unroll
    for (int pr = 0; pr < 4; ++pr) {
      const uint32_t sel = pr | (pr << 4) | ((4 + pr) << 8) | ((4 + pr) << 12);
      const uint32_t t = (prmt(w, w1, sel) & 0x0078000Fu) | kMagic;
      // (h - 128, h / 8 - 16)
      const uint32_t q = bf2_fma(t, 0x3E003F80u, 0xC180C300u);
      h[pr] = bf2_fma(q, s2, b2);
    }
  } else if constexpr (BITS == 2) {
    // byte p holds codes 4p .. 4p+3; pairs (4p, 4p+1) from the byte itself
    // (128 + q, 128 + 4 q) and (4p+2, 4p+3) from the byte two bits down
    // (128 + 4 q, 128 + 16 q)
    const uint32_t w2 = w >> 2;
#pragma unroll
    for (int pr = 0; pr < 4; ++pr) {
      const uint32_t sel = pr | (pr << 4) | (pr << 8) | (pr << 12);
      const uint32_t ta = (prmt(w, w, sel) & 0x000C0003u) | kMagic;
      const uint32_t tb = (prmt(w2, w2, sel) & 0x0030000Cu) | kMagic;
      const uint32_t qa = bf2_fma(ta, 0x3E803F80u, 0xC200C300u);  // (h - 128, h/4 - 32)
      const uint32_t qb = bf2_fma(tb, 0x3D803E80u, 0xC100C200u);  // (h/4 - 32, h/16 - 8)
      h[2 * pr] = bf2_fma(qa, s2, b2);
      h[2 * pr + 1] = bf2_fma(qb, s2, b2);
    }
  } else {
    static_assert(BITS == 8, "2-, 4- and 8-bit codes");
    constexpr uint32_t kF = 0x4B000000u;  // binary32 2^23
    const float2 m2 = make_float2(-8388608.0f, -8388608.0f);
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const uint32_t f0 = prmt(w, kF, 0x7440u | (2 * pr));
      const uint32_t f1 = prmt(w, kF, 0x7440u | (2 * pr + 1));
      const float2 q = __fadd2_rn(make_float2(__uint_as_float(f0), __uint_as_float(f1)), m2);
      h[pr] = bf2_fma(pack_bf16x2(q.x, q.y), s2, b2);
    }
  }
}

template <int BITS, int GS, int MC>
__global__ void __launch_bounds__(qmm_threads<MC>(), 1)
    qmm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s,
               const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_x,
               const QmmParams p) {
  using SH = QmmShape<MC>;
  using ST = QmmStage<BITS>;
  constexpr int CPS = ST::CPS;                       // MMA chunks per stage
  constexpr int SC = ST::SC;                         // codes per stage row
  constexpr int NP = kQmmParts;                      // parts per stage row
  constexpr int NAB = SH::kAbufs;
  constexpr int nw = 4 * NP;                         // dequant warps: 0 .. nw-1
  constexpr uint32_t kStageBytes = ST::bytes;        // codes + scale + bias windows
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = smem_u32(smem);
  // the x slots, then the weight stages, 1024-aligned (1 KB of slack)
  const uint32_t xring = (base + QmmSmem::ring_off + 1023u) & ~1023u;
  const uint32_t wring = xring + static_cast<uint32_t>(p.nxs) * SH::kXBytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem);
  uint64_t *wfull = bars, *wempty = bars + kMmaMaxStages;
  uint64_t *xfull = bars + 2 * kMmaMaxStages, *xempty = xfull + kQmmMaxX;
  uint64_t *abfull = xempty + kQmmMaxX, *abempty = abfull + kQmmMaxAbufs;
  uint64_t *dfull = abempty + kQmmMaxAbufs, *dempty = dfull + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + QmmSmem::tmem_off);
  int *tile_flag = reinterpret_cast<int *>(smem + QmmSmem::flag_off);
  const int nst = p.nst, nxs = p.nxs;
  grid_launch_dependents();

  if (warp == nw) {
    if (lane < nst) {
      mbar_init(&wfull[lane], 1);  // the producer's expect_tx arrival
      mbar_init(&wempty[lane], nw);
    }
    if (lane < nxs) {
      mbar_init(&xfull[lane], 1);
      mbar_init(&xempty[lane], 1);  // tcgen05.commit
    }
    if (lane < NAB) {
      mbar_init(&abfull[lane], qmm_warps_per_chunk<BITS>());
      mbar_init(&abempty[lane], 1);  // tcgen05.commit
    }
    if (lane < 2) {
      mbar_init(&dfull[lane], SH::kIssuers);  // a tcgen05.commit per issuer
      mbar_init(&dempty[lane], nw);  // every dequant warp
    }
    fence_mbar_init();
  }
  if (warp == nw + 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kMmaTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  // every thread's first global access follows: wait for the previous grid
  grid_dependency_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const long long v0 = qmm_start(blockIdx.x, p);
  const long long v1 = qmm_start(blockIdx.x + 1, p);

  if (warp == nw) {
    // ---------------- producer (one thread) ----------------
    if (lane == 0) {
      RingPos sp, xp;
      long long issued = 0, xissued = 0;
      bool dead = false;
      const uint64_t pol_stream = l2_policy_evict_first();  // read once
      const uint64_t pol_keep = l2_policy_evict_last();     // x: read by every tile
      // The two rings advance independently: a weight stage needs its slot
      // back from the dequant warps, an x chunk its slot back from the
      // MMAs.  The thread polls both and issues whatever is free, so the
      // weight stream is never held up behind an x slot.  The bound on
      // consecutive idle polls only ends a broken launch.
      long long wv = v0;                                   // next weight step
      long long xc = 0;                                    // next x chunk of the range
      const long long xn = (v1 - v0) * CPS;
      int wt = static_cast<int>(v0 / p.nstage), wc = static_cast<int>(v0 % p.nstage);
      uint32_t idle = 0;
      while ((wv < v1 || xc < xn) && !dead) {
        bool any = false;
        if (wv < v1 && (issued < nst || mbar_test(&wempty[sp.idx], sp.phase ^ 1u))) {
          const int r0 = (wt / p.nmb) * kMmaRows;
          const uint32_t dst = wring + sp.idx * kStageBytes;
          uint64_t *bar = &wfull[sp.idx];
          mbar_arrive_expect_tx(bar, kStageBytes);
#pragma unroll
          for (int bx = 0; bx < ST::NBOX; ++bx)
            tma_load_2d(dst + bx * (kMmaRows * 128), &tm_w, (wc * ST::NBOX + bx) * 128, r0, bar,
                        pol_stream);
          const int wg = (wc * (SC / GS)) & ~7;
          tma_load_2d(dst + ST::s_off, &tm_s, wg, r0, bar, pol_stream);
          tma_load_2d(dst + ST::b_off, &tm_b, wg, r0, bar, pol_stream);
          sp.next(nst);
          ++issued;
          ++wv;
          if (++wc == p.nstage) {
            wc = 0;
            ++wt;
          }
          any = true;
        }
        if (xc < xn && (xissued < nxs || mbar_test(&xempty[xp.idx], xp.phase ^ 1u))) {
          const long long v = v0 + xc / CPS;
          const int h = static_cast<int>(xc % CPS);
          const int t = static_cast<int>(v / p.nstage), c = static_cast<int>(v % p.nstage);
          const int mb = t % p.nmb;
          const uint32_t dst = xring + xp.idx * SH::kXBytes;
          uint64_t *bar = &xfull[xp.idx];
          mbar_arrive_expect_tx(bar, SH::kXBytes);
          const int k0 = c * SC + h * kMmaKC;
          tma_load_2d(dst, &tm_x, k0, mb * MC, bar, pol_keep);
          tma_load_2d(dst + MC * 128, &tm_x, k0 + 64, mb * MC, bar, pol_keep);
          xp.next(nxs);
          ++xissued;
          ++xc;
          any = true;
        }
        if (any) {
          idle = 0;
        } else if (++idle > (1u << 24)) {
          dead = true;
        } else {
          __nanosleep(16);
        }
      }
      // every copy issued must land before the CTA exits: wait (bounded)
      // for the last phase of each slot in use, the oldest first
      {
        const int inuse = issued < nst ? static_cast<int>(issued) : nst;
        RingPos q = sp;
        q.phase ^= 1u;
        if (issued < nst) q = RingPos();
        for (int i = 0; i < inuse; ++i) {
          if (!dead && !mbar_wait_sleep(&wfull[q.idx], q.phase)) dead = true;
          q.next(nst);
        }
      }
      {
        const int inuse = xissued < nxs ? static_cast<int>(xissued) : nxs;
        RingPos q = xp;
        q.phase ^= 1u;
        if (xissued < nxs) q = RingPos();
        for (int i = 0; i < inuse; ++i) {
          if (!dead && !mbar_wait_sleep(&xfull[q.idx], q.phase)) dead = true;
          q.next(nxs);
        }
      }
      if (dead && p.err) atomicOr(p.err, 2);
    }
    __syncwarp();
  } else if (warp > nw) {
    // ---------------- MMA warps ----------------
    const int issuer = warp - nw - 1;
    RingPos ap, xp;
    int sidx = 0, jj = 0;  // segments done; chunk index inside the segment
    bool dead = false;
    const uint64_t xdesc0 = sw128_desc(xring);
    int c = static_cast<int>(v0 % p.nstage);
    bool seg_start = true;
    uint32_t tmem_d = 0;
    int db = 0;
    for (long long v = v0; v < v1; ++v) {
      if (seg_start) {
        db = sidx & 1;
        jj = 0;
        const uint32_t dph = static_cast<uint32_t>((sidx >> 1) & 1);
        if (sidx >= 2 && !dead && !mbar_wait_sleep(&dempty[db], dph ^ 1u)) dead = true;
        tc_fence_after();
        tmem_d = tmem_base + SH::dcol(db, issuer);
      }
      const bool seg_end = (c == p.nstage - 1) || (v == v1 - 1);
#pragma unroll 1
      for (int h = 0; h < CPS; ++h, ++jj) {
        if (jj % SH::kIssuers != issuer) {  // another issuer's chunk
          ap.next(NAB);
          xp.next(nxs);
          continue;
        }
        if (!dead && !mbar_wait_sleep(&abfull[ap.idx], ap.phase)) dead = true;
        if (!dead && !mbar_wait_sleep(&xfull[xp.idx], xp.phase)) dead = true;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a0 = tmem_base + ap.idx * 64;
          // descriptors advance in 16-byte units inside the start field
          // (shared addresses stay below 2^18): box j / 4 of the chunk,
          // 32 bytes (16 k) per MMA inside the 128-byte swizzled row
          const uint64_t d0 = xdesc0 + static_cast<uint64_t>((xp.idx * SH::kXBytes) >> 4);
          if (jj < SH::kIssuers) {
            // this issuer's first chunk of the segment: its first MMA into
            // each accumulator overwrites it
#pragma unroll
            for (int j = 0; j < kMmaKC / 16; ++j) {
              const uint64_t dj =
                  d0 + static_cast<uint64_t>(((j >> 2) * MC * 128 + (j & 3) * 32) >> 4);
              umma_bf16_ta<MC>(tmem_d + (j % SH::kNacc) * MC, a0 + j * 8, dj,
                               j < SH::kNacc ? 0u : 1u);
            }
          } else {
            umma_chunk_acc<MC>(tmem_d, a0, d0);
          }
          mma_commit(&abempty[ap.idx]);
          mma_commit(&xempty[xp.idx]);
        }
        __syncwarp();
        ap.next(NAB);
        xp.next(nxs);
      }
      // every issuer signals the segment's end, with or without chunks in
      // it (the commit covers all of this thread's earlier MMAs)
      if (seg_end && lane == 0) mma_commit(&dfull[db]);
      __syncwarp();
      if (seg_end) ++sidx;
      seg_start = seg_end;
      if (++c == p.nstage) c = 0;
    }
    if (dead && p.err && lane == 0) atomicOr(p.err, 2);
  } else {
    // ---------------- dequant warps ----------------
    const int r = tid % kMmaRows;
    const int qt = tid / kMmaRows;                   // part of the stage row
    constexpr int QW = ST::SB / 4 / NP;              // words per part
    constexpr int QC = qmm_part_codes<BITS>();       // codes per part
    constexpr int CPW = 32 / BITS;                   // codes per word
    constexpr int HPW = CPW / 2;                     // bf16 pairs per word
    constexpr int NV = QC / 2;                       // tensor-memory columns written
    constexpr int NG = QC >= GS ? QC / GS : 1;       // groups in a part
    const int cc = (qt * QC) / kMmaKC;               // MMA chunk within the stage
    uint32_t woff[QW / 4];  // the part's 16-byte pieces in the swizzled boxes
#pragma unroll
    for (int i = 0; i < QW / 4; ++i) {
      const int pc = (QW / 4) * qt + i;  // 16-byte piece of the row's SB bytes
      woff[i] = (pc / 8) * (kMmaRows * 128) + r * 128 + ((((pc % 8) ^ (r & 7)) & 7) << 4);
    }
    const int gpart = (qt * QC) / GS;  // the part's first group, from the stage's
    const uint32_t wrow = r * 32;
    const uint32_t wswz = static_cast<uint32_t>((r >> 2) & 1);
    const uint32_t lane_q = static_cast<uint32_t>(32 * (warp % 4)) << 16;
    const uint32_t ta0 = tmem_base + lane_q + static_cast<uint32_t>((qt * QC) % kMmaKC) / 2;
    RingPos sp, ap;
    for (int i = 0; i < cc; ++i) ap.next(NAB);
    long long kc = cc;  // MMA chunk count of this thread's chunk
    bool dead = false;
    struct Regs {
      uint32_t wd[QW];
      uint32_t s2[NG], b2[NG];
    };
    auto load = [&](Regs &R, int c) {
      if (!dead && !mbar_wait(&wfull[sp.idx], sp.phase)) dead = true;
      const uint32_t stg = wring + sp.idx * kStageBytes;
#pragma unroll
      for (int i = 0; i < QW / 4; ++i)
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n"
                     : "=r"(R.wd[4 * i]), "=r"(R.wd[4 * i + 1]), "=r"(R.wd[4 * i + 2]),
                       "=r"(R.wd[4 * i + 3])
                     : "r"(stg + woff[i]));
      // NG groups from window index gh (a multiple of NG, so one aligned
      // load); 32-byte swizzle: 16-byte piece j of row r at j ^ ((r / 4) % 2)
      const int gh = ((c * (SC / GS)) & 7) + gpart;
      const uint32_t wo = wrow + ((((2 * gh) >> 4) ^ wswz) << 4) + ((2 * gh) & 15);
      uint32_t sv[(NG + 1) / 2], bv[(NG + 1) / 2];
      lds_groups<NG>(stg + ST::s_off + wo, sv);
      lds_groups<NG>(stg + ST::b_off + wo, bv);
#pragma unroll
      for (int g = 0; g < NG; ++g) {
        const uint32_t sb = (sv[g / 2] >> (16 * (g % 2))) & 0xffffu;
        const uint32_t bb = (bv[g / 2] >> (16 * (g % 2))) & 0xffffu;
        R.s2[g] = sb | (sb << 16);
        R.b2[g] = bb | (bb << 16);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&wempty[sp.idx]);
      sp.next(nst);
    };
    long long v = v0;
    int t = static_cast<int>(v0 / p.nstage), c = static_cast<int>(v0 % p.nstage);
    int cseg0 = c, sidx = 0;
    auto step = [&](Regs &R, Regs &N) {
      // the A buffer must be free: its previous MMAs have completed
      if (kc >= NAB && !dead && !mbar_wait(&abempty[ap.idx], ap.phase ^ 1u)) dead = true;
      tc_fence_after();
      // 32 (or 16) columns at a time: unpack the words behind them, store
      const uint32_t ta = ta0 + ap.idx * 64;
      constexpr int PCOLS = NV < 32 ? NV : 32;
      constexpr int WPP = PCOLS / HPW;  // words per piece
#pragma unroll
      for (int pc = 0; pc < NV / PCOLS; ++pc) {
        uint32_t av[PCOLS];
#pragma unroll
        for (int i = 0; i < WPP; ++i) {
          const int wi = pc * WPP + i;
          const int g = (QC >= GS) ? (wi * CPW) / GS : 0;  // compile time
          uint32_t hw[HPW];
          unpack_word_bf16<BITS>(R.wd[wi], R.s2[g], R.b2[g], hw);
#pragma unroll
          for (int j = 0; j < HPW; ++j) av[i * HPW + j] = hw[j];
        }
        if constexpr (PCOLS == 32)
          tmem_st32(ta + 32 * pc, av);
        else
          tmem_st16(ta + 16 * pc, av);
      }
      // the next stage of this CTA's walk
      const int tc = t;
      const bool seg_end = (c == p.nstage - 1) || (v == v1 - 1);
      const int seg_chunks = (c - cseg0 + 1) * CPS;  // when seg_end: the segment's chunks
      const bool whole_tile = seg_end && cseg0 == 0 && c == p.nstage - 1;
      ++v;
      if (++c == p.nstage) {
        c = 0;
        ++t;
      }
      if (seg_end) cseg0 = c;
      if (v < v1) load(N, c);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&abfull[ap.idx]);
      for (int i = 0; i < CPS; ++i) ap.next(NAB);
      kc += CPS;
      // ---- epilogue of the segment: every dequant warp, its lane quarter
      // of the tile's rows and every (nw / 4)-th piece of 16 columns ----
      if (seg_end) {
        constexpr int NPC = MC / 16;  // 16-column pieces
        constexpr int NEG = nw / 4;   // warps per lane quarter
        const int eg = warp / 4;
        const int db = sidx & 1;
        const uint32_t dph = static_cast<uint32_t>((sidx >> 1) & 1);
        if (!dead && !mbar_wait(&dfull[db], dph)) dead = true;
        tc_fence_after();
        const uint32_t dcol = tmem_base + lane_q + SH::dcol(db, 0);
        // issuers that had chunks in the segment (the others' accumulators
        // hold an older segment)
        const int used = seg_chunks < SH::kIssuers ? seg_chunks : SH::kIssuers;
        const int rt = 32 * (warp % 4) + lane;  // row in the tile
        const int nt = tc / p.nmb, mb = tc - nt * p.nmb;
        const int row = nt * kMmaRows + rt;
        const bool row_ok = row < p.N;
        auto read_piece = [&](int pc, float (&d)[16]) {
          tmem_ld16(dcol + 16 * pc, d);
#pragma unroll
          for (int a = 1; a < SH::kIssuers; ++a) {
            if (a < used) {  // warp-uniform
              float e[16];
              tmem_ld16(dcol + a * MC + 16 * pc, e);
#pragma unroll
              for (int m = 0; m < 16; ++m) d[m] += e[m];
            }
          }
        };
        if (whole_tile) {
#pragma unroll 1
          for (int pc = eg; pc < NPC; pc += NEG) {
            float d[16];
            read_piece(pc, d);
            const int m0 = mb * MC + 16 * pc;
#pragma unroll
            for (int m = 0; m < 16; ++m)
              if (row_ok && m0 + m < p.M)
                p.y[static_cast<size_t>(m0 + m) * p.N + row] = f32_to_bf16(d[m]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&dempty[db]);
        } else {
          // a part of tile tc: leave it in this CTA's slot (0 for the
          // range's first segment, 1 for its last), count it, and if it is
          // the tile's last part to arrive, add all parts in CTA order
          const long long ts = static_cast<long long>(tc) * p.nstage;
          const int first = qmm_owner(ts, p);
          const int last = qmm_owner(ts + p.nstage - 1, p);
          float *mine = p.part + (static_cast<size_t>(blockIdx.x) * 2 + (v0 >= ts ? 0 : 1)) *
                                     (static_cast<size_t>(MC) * kMmaRows);
#pragma unroll 1
          for (int pc = eg; pc < NPC; pc += NEG) {
            float d[16];
            read_piece(pc, d);
#pragma unroll
            for (int m = 0; m < 16; ++m) mine[(16 * pc + m) * kMmaRows + rt] = d[m];
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&dempty[db]);
          __threadfence();
          named_sync(2, nw * 32);
          if (warp == 0 && lane == 0)
            *tile_flag = atomicAdd(&p.cnt[tc], 1) == last - first ? 1 : 0;
          named_sync(2, nw * 32);
          if (*tile_flag) {
            __threadfence();
#pragma unroll 1
            for (int pc = eg; pc < NPC; pc += NEG) {
              float acc[16];
#pragma unroll
              for (int m = 0; m < 16; ++m) acc[m] = 0.f;
              for (int j = first; j <= last; ++j) {
                const long long sj = qmm_start(j, p);
                const float *pj = p.part + (static_cast<size_t>(j) * 2 + (sj >= ts ? 0 : 1)) *
                                               (static_cast<size_t>(MC) * kMmaRows);
#pragma unroll
                for (int m = 0; m < 16; ++m) acc[m] += __ldcg(pj + (16 * pc + m) * kMmaRows + rt);
              }
              const int m0 = mb * MC + 16 * pc;
#pragma unroll
              for (int m = 0; m < 16; ++m)
                if (row_ok && m0 + m < p.M)
                  p.y[static_cast<size_t>(m0 + m) * p.N + row] = f32_to_bf16(acc[m]);
            }
            if (warp == 0 && lane == 0) p.cnt[tc] = 0;  // ready for the next launch
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

namespace qmvq {
namespace {

int say(char *msg, size_t n, int code, const char *fmt, ...) __attribute__((format(printf, 4, 5)));
int say(char *msg, size_t n, int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  if (msg && n) vsnprintf(msg, n, fmt, ap);
  va_end(ap);
  return code;
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// A 2-D row-major tensor [rows][cols] of `esize`-byte elements, row stride
// `stride` bytes, copied in boxes of [box_rows][box_cols].
bool encode_2d(CUtensorMap *map, const void *ptr, CUtensorMapDataType type, uint64_t cols,
               uint64_t rows, uint64_t stride, uint32_t box_cols, uint32_t box_rows,
               CUtensorMapSwizzle swz, CUtensorMapL2promotion l2) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {stride};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, type, 2, const_cast<void *>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, l2, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

template <int BITS, int GS, int MC>
int launch_t(const QmmArgs &a, char *msg, size_t n) {
  using SH = qmvk::QmmShape<MC>;
  constexpr uint32_t kStageBytes = qmvk::QmmStage<BITS>::bytes;
  auto kern = qmvk::qmm_kernel<BITS, GS, MC>;
  qmvk::QmmParams p;
  std::memset(&p, 0, sizeof p);
  p.y = static_cast<uint16_t *>(a.y);
  p.err = a.err;
  p.M = a.M;
  p.N = a.N;
  p.nmb = (a.M + MC - 1) / MC;
  p.nstage = a.K / qmvk::QmmStage<BITS>::SC;
  const long long tiles = static_cast<long long>((a.N + qmvk::kMmaRows - 1) / qmvk::kMmaRows) *
                          p.nmb;
  p.nsteps = tiles * p.nstage;
  p.part = a.part;
  p.cnt = a.cnt;
  p.gran = a.part ? 1 : p.nstage;
  // shared memory: the x slots (about two fifths, at least three), then as
  // many weight stages as fit
  const int room = a.smem_optin - static_cast<int>(qmvk::QmmSmem::ring_off) - 1024;
  int nxs = static_cast<int>((room * 2LL / 5) / SH::kXBytes);
  if (nxs < 3) nxs = 3;
  if (nxs > qmvk::kQmmMaxX) nxs = qmvk::kQmmMaxX;
  int nst = (room - nxs * static_cast<int>(SH::kXBytes)) / static_cast<int>(kStageBytes);
  if (nst > qmvk::kMmaMaxStages) nst = qmvk::kMmaMaxStages;
  if (nst < 2) return say(msg, n, QMV_ERR_UNSUPPORTED, "qmm: shared memory too small");
  p.nst = nst;
  p.nxs = nxs;
  const int smem = static_cast<int>(qmvk::QmmSmem::ring_off) + 1024 +
                   nxs * static_cast<int>(SH::kXBytes) + nst * static_cast<int>(kStageBytes);
  const uint32_t row_bytes = static_cast<uint32_t>(static_cast<long long>(a.K) * BITS / 8);
  const int G = a.K / GS;
  CUtensorMap tw, ts, tb, tx;
  if (!encode_2d(&tw, a.w, CU_TENSOR_MAP_DATA_TYPE_UINT8, row_bytes, a.N, row_bytes, 128,
                 qmvk::kMmaRows, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
      !encode_2d(&ts, a.scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, G, a.N, 2ull * G,
                 qmvk::kMmaWinGroups, qmvk::kMmaRows, CU_TENSOR_MAP_SWIZZLE_32B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_128B) ||
      !encode_2d(&tb, a.biases, CU_TENSOR_MAP_DATA_TYPE_UINT16, G, a.N, 2ull * G,
                 qmvk::kMmaWinGroups, qmvk::kMmaRows, CU_TENSOR_MAP_SWIZZLE_32B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_128B) ||
      !encode_2d(&tx, a.x, CU_TENSOR_MAP_DATA_TYPE_UINT16, a.K, a.M, 2ull * a.K, 64, MC,
                 CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B))
    return say(msg, n, QMV_ERR_CUDA, "qmm: cuTensorMapEncodeTiled failed");
  int d = 0;
  cudaGetDevice(&d);
  static int granted[64] = {};
  if (d >= 0 && d < 64 && smem > granted[d]) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, a.smem_optin);
    if (e != cudaSuccess)
      return say(msg, n, QMV_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    granted[d] = a.smem_optin;
  }
  const long long grid = tiles * p.nstage < a.sms ? tiles * p.nstage : a.sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.part ? grid : (tiles < a.sms ? tiles : a.sms)));
  cfg.blockDim = dim3(qmvk::qmm_threads<MC>());
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t le = cudaLaunchKernelEx(&cfg, kern, tw, ts, tb, tx, p);
  if (le != cudaSuccess) {
    cudaGetLastError();  // clear it
    return say(msg, n, QMV_ERR_CUDA, "qmm launch: %s", cudaGetErrorString(le));
  }
  return 0;
}

template <int BITS, int GS>
int launch_c(const QmmArgs &a, char *msg, size_t n) {
  switch (qmm_cols(a.M)) {
    case 16: return launch_t<BITS, GS, 16>(a, msg, n);
    case 32: return launch_t<BITS, GS, 32>(a, msg, n);
    case 64: return launch_t<BITS, GS, 64>(a, msg, n);
    default: return launch_t<BITS, GS, 128>(a, msg, n);
  }
}

template <int BITS>
int launch_g(const QmmArgs &a, char *msg, size_t n) {
  switch (a.gs) {
    case 32: return launch_c<BITS, 32>(a, msg, n);
    case 64: return launch_c<BITS, 64>(a, msg, n);
    case 128: return launch_c<BITS, 128>(a, msg, n);
    default: return say(msg, n, QMV_ERR_UNSUPPORTED, "qmm: group_size=%d", a.gs);
  }
}

}  // namespace

int qmm_stage_codes(int bits) {
  switch (bits) {
    case 2: return qmvk::QmmStage<2>::SC;
    case 4: return qmvk::QmmStage<4>::SC;
    case 8: return qmvk::QmmStage<8>::SC;
    default: return 0;
  }
}

int qmm_cols(int M) { return M <= 16 ? 16 : (M <= 32 ? 32 : (M <= 64 ? 64 : 128)); }

long long qmm_tiles(int M, int N) {
  const int mc = qmm_cols(M);
  return static_cast<long long>((N + qmvk::kMmaRows - 1) / qmvk::kMmaRows) * ((M + mc - 1) / mc);
}

size_t qmm_part_bytes(int M, int sms) {
  return static_cast<size_t>(sms) * 2 * qmm_cols(M) * qmvk::kMmaRows * sizeof(float);
}

int qmm_launch(const QmmArgs &a, char *msg, size_t n) {
  switch (a.bits) {
    case 2: return launch_g<2>(a, msg, n);
    case 4: return launch_g<4>(a, msg, n);
    case 8: return launch_g<8>(a, msg, n);
    default: return say(msg, n, QMV_ERR_UNSUPPORTED, "qmm: bits=%d", a.bits);
  }
}

}  // namespace qmvq
