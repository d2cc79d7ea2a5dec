// qmv_qvm.cuh -- the non-transposed product y = x @ dequant(W) (the pages'
// qvm: "mlx/include/mlx/backend/metal/kernels/quantized.h", qvm_impl and
// affine_qvm, MLX 0.30.1).  W has K rows of N codes each (the same packed
// row format as qmv's weights), and its groups run along N: row k, codes
// [g*gs, (g+1)*gs) share scale[k][g] and bias[k][g].
//
//   y[m][n] = sum_k x[m][k] * (scale[k][n/gs] * q[k][n] + bias[k][n/gs])
//
// A lane owns a chunk of 8 consecutive columns (8 codes: `bits` bytes of a
// row) and walks rows; a warp's 32 chunks are 256 consecutive columns, so
// each row read is one contiguous segment.  The rows are split between the
// 8 CTAs of a thread-block cluster that share a 256-column block, and
// between the warps of each CTA.  Per row a lane forms xs = x * scale,
// turns its 8 codes into exact floats (2^23 + q from the bits, minus 2^23)
// and accumulates xs * q per column with paired fp32 FMAs, and x * bias once
// for its group.  The partials are added in a fixed order: over a CTA's
// warps through shared memory, then over the cluster's CTAs through
// distributed shared memory by the cluster's first CTA, which rounds once to
// bf16 and stores.  No global scratch, no atomics: the result does not
// depend on timing.
#pragma once

#include <cooperative_groups.h>

#include "qmv_device.cuh"
#include "qmv_mma.cuh"

namespace qmvk {

constexpr int kQvmCluster = 8;     // CTAs sharing a column block (row split)
constexpr int kQvmWarps = 16;      // warps per CTA (row split)
constexpr int kQvmCols = 256;      // columns per block: 32 lanes x 8 codes
constexpr int kQvmUnroll = 8;      // rows per block of loads (two blocks in flight)

struct QvmParams {
  const uint8_t *w;       // packed rows [K][row_bytes]
  const uint16_t *s, *b;  // bf16 [K][G]
  const uint16_t *x;      // bf16 [M][K]
  uint16_t *y;            // bf16 [M][N]
  int M, K, N, G;
  int gs_shift;           // log2(group size)
  uint32_t row_bytes;     // N * bits / 8
};

// The 8 codes of chunk c of a row: bytes [c * BITS, c * BITS + BITS), read
// as the aligned words that hold them (never a word past the row's bytes:
// the row length is a whole number of words).
template <int BITS>
__device__ __forceinline__ uint64_t qvm_chunk(const uint8_t *row, int c) {
  const uint32_t byte0 = static_cast<uint32_t>(c) * BITS;
  const uint32_t *wp = reinterpret_cast<const uint32_t *>(row) + (byte0 >> 2);
  const int off = static_cast<int>(byte0 & 3);
  uint64_t v = __ldg(wp);
  if (off + BITS > 4) v |= static_cast<uint64_t>(__ldg(wp + 1)) << 32;
  return v >> (8 * off);
}

// One row of a lane's chunk: acc[j] += xs * (q[2j], q[2j+1]).  Codes become
// exact floats from their bits under the binary32 exponent of 2^23 (2^23 + v
// minus 2^23).  For 2-, 4- and 8-bit codes each byte of the chunk is shifted
// down once and its codes are masked in place: a code 2^i bits up in its
// byte comes out as 2^i * q, which the matching pre-divided multiplier
// xs * 2^-i (exact) undoes.
template <int BITS>
__device__ __forceinline__ void qvm_row(uint64_t v, float xs, float2 (&acc)[4]) {
  const float2 m2 = make_float2(-8388608.0f, -8388608.0f);
  if constexpr (BITS == 2 || BITS == 4 || BITS == 8) {
    constexpr int CPB = 8 / BITS;                  // codes per byte
    // the chunk's BITS bytes as 32-bit words (two for 8-bit codes)
    const uint32_t wv[2] = {static_cast<uint32_t>(v), static_cast<uint32_t>(v >> 32)};
    float mul[CPB];
#pragma unroll
    for (int i = 0; i < CPB; ++i) mul[i] = xs * (1.0f / static_cast<float>(1 << (BITS * i)));
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c0 = 2 * j, c1 = 2 * j + 1;        // codes of the pair
      const int y0 = c0 / CPB, y1 = c1 / CPB;      // bytes of the pair's codes
      const uint32_t b0 = wv[y0 / 4] >> (8 * (y0 % 4)), b1 = wv[y1 / 4] >> (8 * (y1 % 4));
      const uint32_t f0 = (b0 & (((1u << BITS) - 1u) << (BITS * (c0 % CPB)))) | 0x4b000000u;
      const uint32_t f1 = (b1 & (((1u << BITS) - 1u) << (BITS * (c1 % CPB)))) | 0x4b000000u;
      const float2 qf = __fadd2_rn(make_float2(__uint_as_float(f0), __uint_as_float(f1)), m2);
      acc[j] = __ffma2_rn(qf, make_float2(mul[c0 % CPB], mul[c1 % CPB]), acc[j]);
    }
  } else {
    const float2 xs2 = make_float2(xs, xs);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t q0 = static_cast<uint32_t>(v >> (BITS * 2 * j)) & ((1u << BITS) - 1u);
      const uint32_t q1 = static_cast<uint32_t>(v >> (BITS * (2 * j + 1))) & ((1u << BITS) - 1u);
      const float2 qf = __fadd2_rn(
          make_float2(__uint_as_float(0x4b000000u | q0), __uint_as_float(0x4b000000u | q1)), m2);
      acc[j] = __ffma2_rn(qf, xs2, acc[j]);
    }
  }
}

template <int BITS>
__global__ void __cluster_dims__(1, kQvmCluster, 1) __launch_bounds__(kQvmWarps * 32, 1)
    qvm_kernel(const QvmParams p) {
  namespace cg = cooperative_groups;
  __shared__ float red[kQvmWarps][kQvmCols];
  __shared__ float part[kQvmCols];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = blockIdx.x, rank = blockIdx.y, m = blockIdx.z;
  const int c = nb * 32 + lane;              // this lane's chunk of 8 columns
  const bool live = 8 * c < p.N;
  const int k0 = static_cast<int>(static_cast<long long>(p.K) * rank / kQvmCluster);
  const int k1 = static_cast<int>(static_cast<long long>(p.K) * (rank + 1) / kQvmCluster);
  const uint16_t *xr = p.x + static_cast<size_t>(m) * p.K;
  const int g = (8 * c) >> p.gs_shift;       // the chunk's group (one per chunk)
  grid_launch_dependents();
  grid_dependency_wait();

  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};
  float bacc = 0.f;
  // A warp takes rows k0 + warp, k0 + warp + 16, ... in blocks of kQvmUnroll;
  // the next block's loads are in flight while the current one is computed.
  struct Block {
    uint64_t v[kQvmUnroll];
    uint32_t s[kQvmUnroll], b[kQvmUnroll], x[kQvmUnroll];
  };
  auto load = [&](int kb, Block &blk) {
#pragma unroll
    for (int u = 0; u < kQvmUnroll; ++u) {
      const int k = kb + u * kQvmWarps;
      const int kk = k < k1 ? k : kb;  // a valid row; its terms are dropped below
      blk.v[u] = qvm_chunk<BITS>(p.w + static_cast<size_t>(kk) * p.row_bytes, c);
      blk.s[u] = __ldg(p.s + static_cast<size_t>(kk) * p.G + g);
      blk.b[u] = __ldg(p.b + static_cast<size_t>(kk) * p.G + g);
      blk.x[u] = k < k1 ? __ldg(xr + kk) : 0u;  // x = +0: the row adds nothing
    }
  };
  constexpr int kStep = kQvmWarps * kQvmUnroll;
  if (live && k0 + warp < k1) {
    Block cur, nxt;
    load(k0 + warp, cur);
    for (int kb = k0 + warp; kb < k1; kb += kStep) {
      if (kb + kStep < k1) load(kb + kStep, nxt);
#pragma unroll
      for (int u = 0; u < kQvmUnroll; ++u) {
        const float xk = bf16_to_f32(static_cast<uint16_t>(cur.x[u]));
        const float xs = xk * bf16_to_f32(static_cast<uint16_t>(cur.s[u]));
        bacc = fmaf(xk, bf16_to_f32(static_cast<uint16_t>(cur.b[u])), bacc);
        qvm_row<BITS>(cur.v[u], xs, acc);
      }
      cur = nxt;
    }
  }
  // columns of this warp's partials, then the CTA's sum in warp order
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    red[warp][8 * lane + 2 * j] = acc[j].x + bacc;
    red[warp][8 * lane + 2 * j + 1] = acc[j].y + bacc;
  }
  __syncthreads();
  for (int col = threadIdx.x; col < kQvmCols; col += blockDim.x) {
    float sum = 0.f;
    for (int w = 0; w < kQvmWarps; ++w) sum += red[w][col];
    part[col] = sum;
  }
  // the cluster's partials, added by its first CTA in rank order
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();
  if (rank == 0) {
    for (int col = threadIdx.x; col < kQvmCols; col += blockDim.x) {
      const int n = nb * kQvmCols + col;
      float sum = 0.f;
      for (int r = 0; r < kQvmCluster; ++r) sum += cluster.map_shared_rank(part, r)[col];
      if (n < p.N) p.y[static_cast<size_t>(m) * p.N + n] = f32_to_bf16(sum);
    }
  }
  cluster.sync();  // the other CTAs keep their shared memory until it was read
}

// ---------------------------------------------------------------------------
// The staged form (row strides a multiple of 16 bytes): the same lanes,
// column blocks and cluster row split, with the rows streamed into shared
// memory by the tensor-copy engine.  A CTA's rows are one contiguous range;
// per stage one thread copies kQvtRows rows of the block's 32 * BITS bytes
// (2-D box, rows past K arrive as zeros) and the rows' 16-byte scale and
// bias windows (8 groups from the block's first group rounded down to a
// multiple of 8); sixteen consumer warps take the stage's rows in turn.
// Long copies of many rows keep enough bytes in flight to stream at HBM
// speed, where per-lane loads of a few bytes per row did not.
// ---------------------------------------------------------------------------
constexpr int kQvtRows = 64;    // rows per stage
constexpr int kQvtWarps = 16;   // consumer warps
constexpr int kQvtStages = 8;   // stages in the ring

struct QvtParams {
  uint16_t *y;            // bf16 [M][N]
  const uint16_t *x;      // bf16 [M][K]
  int *err;               // OR 2 when a bounded wait gave up
  int M, K, N;
  int gs_shift;           // log2(group size)
  uint32_t stage_bytes;   // W rows, then the scale and bias windows
  uint32_t x_off;         // smem offset of the CTA's activations (fp32)
  uint32_t ring_off;      // smem offset of the stages (rounded up to 128 in the kernel)
};

// The cluster (its size set at launch: gridDim.y CTAs share a column block)
template <int BITS>
__global__ void __launch_bounds__((kQvtWarps + 1) * 32, 1)
    qvm_tma_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s,
                   const __grid_constant__ CUtensorMap tm_b, const QvtParams p) {
  namespace cg = cooperative_groups;
  constexpr int WB = 32 * BITS;                     // bytes of a row in the block
  constexpr uint32_t kSOff = kQvtRows * WB;         // scale windows [rows][16 B]
  constexpr uint32_t kBOff = kSOff + kQvtRows * 16; // bias windows
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ float red[kQvtWarps][kQvmCols];
  __shared__ float part[kQvmCols];
  __shared__ uint64_t bars[2 * kQvtStages];
  uint64_t *full = bars, *empty = bars + kQvtStages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = blockIdx.x, rank = blockIdx.y, m = blockIdx.z;
  const int c = nb * 32 + lane;               // this lane's chunk of 8 columns
  const bool live = 8 * c < p.N;
  const int ncl = static_cast<int>(gridDim.y);  // CTAs of the cluster (row split)
  const int k0 = static_cast<int>(static_cast<long long>(p.K) * rank / ncl);
  const int k1 = static_cast<int>(static_cast<long long>(p.K) * (rank + 1) / ncl);
  const int nstg = (k1 - k0 + kQvtRows - 1) / kQvtRows;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t ring = (sbase + p.ring_off + 127u) & ~127u;  // 128 bytes of slack
  float *xs = reinterpret_cast<float *>(smem + p.x_off);
  const int gwin = ((nb * kQvmCols) >> p.gs_shift) & ~7;  // first group of the windows
  grid_launch_dependents();
  if (warp == kQvtWarps) {
    if (lane < kQvtStages) {
      mbar_init(&full[lane], 1);
      mbar_init(&empty[lane], kQvtWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  grid_dependency_wait();

  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};
  float bacc = 0.f;
  bool dead = false;
  if (warp == kQvtWarps) {
    // ---- producer (one thread) ----
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      for (int j = 0; j < nstg; ++j) {
        const int slot = j % kQvtStages;
        if (j >= kQvtStages && !dead &&
            !mbar_wait_sleep(&empty[slot], static_cast<uint32_t>(((j / kQvtStages) - 1) & 1)))
          dead = true;
        const uint32_t dst = ring + slot * p.stage_bytes;
        mbar_arrive_expect_tx(&full[slot], p.stage_bytes);
        const int kr = k0 + j * kQvtRows;
        tma_load_2d(dst, &tm_w, nb * WB, kr, &full[slot], pol);
        tma_load_2d(dst + kSOff, &tm_s, gwin, kr, &full[slot], pol);
        tma_load_2d(dst + kBOff, &tm_b, gwin, kr, &full[slot], pol);
      }
      // every copy lands before the CTA exits
      for (int j = nstg - kQvtStages < 0 ? 0 : nstg - kQvtStages; j < nstg; ++j)
        if (!dead && !mbar_wait_sleep(&full[j % kQvtStages],
                                      static_cast<uint32_t>((j / kQvtStages) & 1)))
          dead = true;
      if (dead && p.err) atomicOr(p.err, 2);
    }
    __syncwarp();
  } else {
    // ---- consumers: the CTA's activations, then the stages ----
    const uint16_t *xr = p.x + static_cast<size_t>(m) * p.K;
    for (int k = k0 + static_cast<int>(threadIdx.x); k < k1; k += kQvtWarps * 32)
      xs[k - k0] = bf16_to_f32(xr[k]);
    named_sync(1, kQvtWarps * 32);
    const int gl = ((8 * c) >> p.gs_shift) - gwin;  // the chunk's group in the window
    const uint32_t cb = static_cast<uint32_t>(lane) * BITS;  // the chunk's bytes in a row
    for (int j = 0; j < nstg; ++j) {
      const int slot = j % kQvtStages;
      if (!dead && !mbar_wait(&full[slot], static_cast<uint32_t>((j / kQvtStages) & 1)))
        dead = true;
      const uint32_t stg = ring + slot * p.stage_bytes;
      const int kr = k0 + j * kQvtRows;
      if (live) {
#pragma unroll 4
        for (int r = warp; r < kQvtRows; r += kQvtWarps) {
          const int k = kr + r;
          if (k >= k1) break;
          const uint32_t ra = stg + static_cast<uint32_t>(r) * WB;
          // the chunk's BITS bytes as the aligned words that hold them
          const uint32_t a0 = ra + (cb & ~3u);
          uint64_t v = lds32(a0);
          if ((cb & 3u) + BITS > 4) v |= static_cast<uint64_t>(lds32(a0 + 4)) << 32;
          v >>= 8 * (cb & 3u);
          const float xk = xs[k - k0];
          const float sk = bf16_to_f32(static_cast<uint16_t>(lds16(stg + kSOff + r * 16 + 2 * gl)));
          const float bk = bf16_to_f32(static_cast<uint16_t>(lds16(stg + kBOff + r * 16 + 2 * gl)));
          bacc = fmaf(xk, bk, bacc);
          qvm_row<BITS>(v, xk * sk, acc);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
    if (dead && p.err && lane == 0) atomicOr(p.err, 2);
  }
  // columns of this warp's partials, then the CTA's sum in warp order
  if (warp < kQvtWarps) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      red[warp][8 * lane + 2 * j] = acc[j].x + bacc;
      red[warp][8 * lane + 2 * j + 1] = acc[j].y + bacc;
    }
  }
  __syncthreads();
  for (int col = threadIdx.x; col < kQvmCols; col += blockDim.x) {
    float sum = 0.f;
    for (int w = 0; w < kQvtWarps; ++w) sum += red[w][col];
    part[col] = sum;
  }
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();
  if (rank == 0) {
    for (int col = threadIdx.x; col < kQvmCols; col += blockDim.x) {
      const int n = nb * kQvmCols + col;
      float sum = 0.f;
      for (int r = 0; r < ncl; ++r) sum += cluster.map_shared_rank(part, r)[col];
      if (n < p.N) p.y[static_cast<size_t>(m) * p.N + n] = f32_to_bf16(sum);
    }
  }
  cluster.sync();
}

}  // namespace qmvk
