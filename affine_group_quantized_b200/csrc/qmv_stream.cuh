// qmv_stream.cuh -- the persistent weight-streaming GEMV kernel (CUDA cores).
//
// One CTA per SM with two warp roles:
//   * consumer warps: each thread owns one 32-code "unit" column of the
//     weight rows and a row phase.  It streams its unit of its rows from HBM
//     with asynchronous 16-byte copies (cp.async) into its own slots of a
//     shared-memory ring several tiles deep; a warp's copies of one row are
//     32 consecutive units (one contiguous 512-byte span at 4 bits).  Each
//     thread reads back only what it copied itself, so no barrier is needed
//     between copy and use: cp.async.wait_group per thread.  Codes are decoded in registers and multiplied with the unit's
//     activations (8-bit integer dot products for 2/4/8-bit codes, fp32 FMAs
//     for 3/5/6-bit codes), the group scale and bias are applied, and the warp
//     reduces the row partials with shuffles into a small shared ring;
//   * one epilogue warp: adds the per-warp partials of each output in a fixed
//     order, adds the residual if any, rounds once to bf16 and stores.
// Consumers and the epilogue hand ring slots over with mbarriers; consumer
// warps never wait for each other.
//
// The same kernel serves every entry point through `mode`:
//   MODE_QMV      y = x @ dequant(W).T
//   MODE_GATE_UP  two weight matrices (gate, up) over one x, one launch
//   MODE_SILU     input v = silu(gate) * up built in fp32; epilogue adds x_resid
//   MODE_GATHER   pairs grouped by expert inside the kernel; every touched
//                 expert's rows are streamed and dotted with all the x rows
//                 routed to it
//
// Work is a list of "segments", each one weight matrix (or expert) paired
// with up to MR activation rows; a segment's N rows are cut into tiles of
// RT rows.  Each CTA owns a contiguous range of the (segment, row) space.
#pragma once

#include "qmv_device.cuh"

namespace qmvk {

enum Mode : int { MODE_QMV = 0, MODE_GATE_UP = 1, MODE_SILU = 2, MODE_GATHER = 3 };

struct StreamParams {
  const uint8_t *w[2];    // packed rows (matrix 0/1); gather: [E*N] rows
  const uint16_t *s[2];   // scales  bf16 [rows, G]
  const uint16_t *b[2];   // biases  bf16 [rows, G]
  uint16_t *y[2];         // outputs bf16
  const uint16_t *x;      // bf16 [M or num_x_rows, K]; MODE_SILU: gate
  const uint16_t *up;     // MODE_SILU: up [M, K]
  const uint16_t *resid;  // MODE_SILU: x_resid [M, N] or null
  const uint32_t *lhs;    // MODE_GATHER: x row of each pair (null: identity)
  const uint32_t *rhs;    // MODE_GATHER: expert of each pair
  int *status;            // MODE_GATHER: OR 1 on an out-of-range index
  int *err;               // OR 2 when a bounded wait gave up (null: none)
  int mode;
  int M;                  // x rows (qmv / gate_up / silu)
  int N, K, G;            // rows per matrix, columns, groups per row
  int gs_shift;           // log2(group_size / 32): unit -> group
  int U, Upad;            // units per row (K/32) and padded count (>= 32)
  int PH;                 // row phases: Upad threads per row, PH rows at once
  int RT;                 // rows per tile = RPT * PH (RPT fixed per kernel)
  int nmat;               // weight matrices (1, or 2 for gate/up)
  int nch;                // activation chunks per matrix: ceil(M / MR)
  int nred;               // slots in the partial-sum ring
  int wpr;                // partial-sum slots per row (consumer warps per row)
  uint32_t row_bytes;     // K * bits / 8
  int num_pairs, num_x_rows, num_experts;
  uint32_t red_off;       // smem offset of the partial-sum ring
  uint32_t red_slot;      // bytes of one ring slot
  uint32_t bar_off;       // smem offset of the ring's mbarriers
  uint32_t grp_off;       // smem offset of the gather grouping tables
  uint32_t cp_off;        // smem offset of the copy ring
  int depth;              // tiles in the copy ring
  int sb_pairs;           // scales/biases copied as aligned 4-byte pairs (G even)
};

// ---------------------------------------------------------------------------
// Tiles and the stage ring, walked with incremental 32-bit bookkeeping.
// Producer, consumers and epilogue run the same walk, so they agree on every
// tile without communicating.
// ---------------------------------------------------------------------------
struct Tile {
  int seg;    // segment index
  int row;    // first row inside the segment's matrix
  int nrows;  // rows in the tile
};

struct TileWalker {
  int seg, row, left, N, RT;
  int stages, st;
  uint32_t phase;

  __device__ __forceinline__ void init(long long v0, long long v1, int N_,
                                       int RT_, int stages_) {
    N = N_;
    RT = RT_;
    stages = stages_;
    seg = static_cast<int>(v0 / N);
    row = static_cast<int>(v0 - static_cast<long long>(seg) * N);
    left = static_cast<int>(v1 - v0);
    st = 0;
    phase = 0;
  }
  __device__ __forceinline__ bool next(Tile &t) {
    if (left <= 0) return false;
    int n = RT < N - row ? RT : N - row;
    n = n < left ? n : left;
    t.seg = seg;
    t.row = row;
    t.nrows = n;
    row += n;
    left -= n;
    if (row == N) {
      row = 0;
      ++seg;
    }
    return true;
  }
  __device__ __forceinline__ void advance_slot() {
    if (++st == stages) {
      st = 0;
      phase ^= 1u;
    }
  }
};

// ---------------------------------------------------------------------------
// Gather grouping (MODE_GATHER), computed redundantly by every CTA from the
// index arrays (a few hundred bytes): a stable counting sort of the pairs by
// expert, then the segment list: each touched expert, in ascending order, with
// its pairs cut into chunks of MR.
// ---------------------------------------------------------------------------
struct Groups {
  int *cnt;        // [E]  valid pairs per expert
  int *off;        // [E]  exclusive prefix of cnt
  int *pairs;      // [P]  pair ids, stably ordered by expert
  int *seg_e;      // [P]  expert of segment s
  int *seg_first;  // [P]  first position in `pairs` of segment s
  int *nseg;       // [1]
};

__device__ __forceinline__ Groups groups_at(unsigned char *smem,
                                           const StreamParams &p) {
  Groups g;
  int *base = reinterpret_cast<int *>(smem + p.grp_off);
  const int E = p.num_experts, P = p.num_pairs;
  g.cnt = base;
  g.off = base + E;
  g.pairs = base + 2 * E;
  g.seg_e = base + 2 * E + P;
  g.seg_first = base + 2 * E + 2 * P;
  g.nseg = base + 2 * E + 3 * P;
  return g;
}

template <int MR>
__device__ void build_groups(const StreamParams &p, Groups g, int tid,
                             int nthreads) {
  const int E = p.num_experts, P = p.num_pairs;
  for (int e = tid; e < E; e += nthreads) g.cnt[e] = 0;
  __syncthreads();
  bool bad = false;
  for (int i = tid; i < P; i += nthreads) {
    const uint32_t e = p.rhs[i];
    const uint32_t xr = p.lhs ? p.lhs[i] : static_cast<uint32_t>(i);
    if (e < static_cast<uint32_t>(E) && xr < static_cast<uint32_t>(p.num_x_rows))
      atomicAdd(&g.cnt[e], 1);
    else
      bad = true;
  }
  if (bad && p.status && blockIdx.x == 0) atomicOr(p.status, 1);
  __syncthreads();
  if (tid < 32) {
    const unsigned full = 0xffffffffu;
    // exclusive scans of the pair counts and of the chunk counts
    int run = 0, srun = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + tid;
      const int c = e < E ? g.cnt[e] : 0;
      const int nc = (c + MR - 1) / MR;
      int incl = c, sincl = nc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(full, incl, o);
        const int ts = __shfl_up_sync(full, sincl, o);
        if (tid >= o) {
          incl += t;
          sincl += ts;
        }
      }
      if (e < E) {
        const int off = run + incl - c;
        const int s0 = srun + sincl - nc;
        g.off[e] = off;
        for (int k = 0; k < nc; ++k) {
          g.seg_e[s0 + k] = e;
          g.seg_first[s0 + k] = off + k * MR;
        }
      }
      run += __shfl_sync(full, incl, 31);
      srun += __shfl_sync(full, sincl, 31);
    }
    if (tid == 0) *g.nseg = srun;
    __syncwarp();
    // stable scatter: pairs in increasing id order, 32 at a time; cnt is
    // reused as the per-expert cursor and ends equal to the count again
    for (int e = tid; e < E; e += 32) g.cnt[e] = 0;
    __syncwarp();
    for (int base = 0; base < P; base += 32) {
      const int i = base + tid;
      int e = -1;
      if (i < P) {
        const uint32_t ee = p.rhs[i];
        const uint32_t xr = p.lhs ? p.lhs[i] : static_cast<uint32_t>(i);
        if (ee < static_cast<uint32_t>(E) &&
            xr < static_cast<uint32_t>(p.num_x_rows))
          e = static_cast<int>(ee);
      }
      const unsigned same = __match_any_sync(full, e);
      const int rank = __popc(same & ((1u << tid) - 1u));
      const int leader = __ffs(same) - 1;
      int cur = 0;
      if (e >= 0 && tid == leader) cur = g.cnt[e];
      cur = __shfl_sync(full, cur, leader);
      if (e >= 0) g.pairs[g.off[e] + cur + rank] = i;
      __syncwarp();
      if (e >= 0 && tid == leader) g.cnt[e] = cur + __popc(same);
      __syncwarp();
    }
  }
  __syncthreads();
}

// What a segment is: the weight array it streams, its activation rows and
// where its outputs go.
struct Seg {
  int arr;    // weight matrix (0/1) or expert index (gather)
  int first;  // first activation row (dense) or first position in pairs
  int count;  // activation rows in this segment (1..MR)
  int key;    // identifies the activation rows (for register reuse)
};

template <int MR>
__device__ __forceinline__ Seg seg_info(const StreamParams &p, const Groups &g,
                                        int s) {
  Seg r;
  if (p.mode == MODE_GATHER) {
    const int e = g.seg_e[s];
    r.arr = e;
    r.first = g.seg_first[s];
    const int end = g.off[e] + g.cnt[e];
    r.count = end - r.first < MR ? end - r.first : MR;
    r.key = r.first;
  } else {
    const int mat = p.nch == 1 ? s : s / p.nch;
    const int c = s - mat * p.nch;
    r.arr = mat;
    r.first = c * MR;
    r.count = p.M - r.first < MR ? p.M - r.first : MR;
    r.key = c;
  }
  return r;
}

// activation row of slot m of a segment (-1 if absent)
template <int MR>
__device__ __forceinline__ int seg_xrow(const StreamParams &p, const Groups &g,
                                        const Seg &sg, int m) {
  if (m >= sg.count) return -1;
  if (p.mode == MODE_GATHER) {
    const int pr = g.pairs[sg.first + m];
    return p.lhs ? static_cast<int>(p.lhs[pr]) : pr;
  }
  return sg.first + m;
}

// Row of the weight arrays that row `row` of segment `arr` lives in.
__device__ __forceinline__ long long abs_row(const StreamParams &p, int arr,
                                           int row) {
  return p.mode == MODE_GATHER ? static_cast<long long>(arr) * p.N + row
                               : static_cast<long long>(row);
}

// ---------------------------------------------------------------------------
// Epilogue warp: sums the consumer warps' partials of each output in a fixed
// order, adds the residual, rounds once to bf16 and stores.
// ---------------------------------------------------------------------------
template <int MR>
__device__ void epilogue_loop(const StreamParams &p, unsigned char *smem,
                              uint64_t *redfull, uint64_t *redempty,
                              const Groups &g, long long v0, long long v1,
                              int lane) {
  TileWalker tw;
  tw.init(v0, v1, p.N, p.RT, p.nred);
  Tile t;
  while (tw.next(t)) {
    const int st = tw.st;
    if (!mbar_wait(&redfull[st], tw.phase)) {
      if (p.err) atomicOr(p.err, 2);
      return;
    }
    const Seg sg = seg_info<MR>(p, g, t.seg);
    const float *rb =
        reinterpret_cast<const float *>(smem + p.red_off + st * p.red_slot);
    for (int o = lane; o < t.nrows * MR; o += 32) {
      const int r = o / MR, m = o % MR;
      if (m < sg.count) {
        float acc = 0.f;
        for (int w = 0; w < p.wpr; ++w) acc += rb[(r * MR + m) * p.wpr + w];
        const int n = t.row + r;
        if (p.mode == MODE_GATHER) {
          const int pr = g.pairs[sg.first + m];
          p.y[0][static_cast<size_t>(pr) * p.N + n] = f32_to_bf16(acc);
        } else {
          const size_t yo = static_cast<size_t>(sg.first + m) * p.N + n;
          if (p.mode == MODE_SILU && p.resid) acc += bf16_to_f32(p.resid[yo]);
          p.y[sg.arr][yo] = f32_to_bf16(acc);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&redempty[st]);
    tw.advance_slot();
  }
}

// ---------------------------------------------------------------------------
// Consumers
// ---------------------------------------------------------------------------

// Asynchronous global -> shared copies of 16, 8 or 4 bytes (cp.async).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(dst), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(a));
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

// Layout of one thread's copy of one row in the ring: the unit's bytes in
// "planes" of 16, 8 or 4 bytes (the largest that divides the unit), each
// plane of all consumer threads contiguous, so that the reads of a warp hit
// 32 consecutive 16/8/4-byte slots (no bank conflicts); then the scale and
// the bias, each as the aligned 4-byte pair that holds it (or the value
// itself when the pairs are not 4-byte aligned).
template <int BITS>
struct CopyLayout {
  static constexpr int kUnitBytes = 4 * BITS;
  static constexpr int kPlane = BITS % 4 == 0 ? 16 : (BITS % 2 == 0 ? 8 : 4);
  static constexpr int kPlanes = kUnitBytes / kPlane;
  // bytes of one row of the ring for Tc threads
  static __host__ __device__ constexpr uint32_t row_bytes(int tc) {
    return static_cast<uint32_t>(tc) * (kUnitBytes + 8);
  }
};

// Issue the copies of the thread's rows of one tile into ring stage `stage`.
template <int BITS, int RPT>
__device__ __forceinline__ void issue_tile(const StreamParams &p, const Tile &t,
                                           int arr, int w_arr, int ph, int u,
                                           int tid, int Tc, uint32_t stage_base) {
  using CL = CopyLayout<BITS>;
  const long long r0 = abs_row(p, arr, t.row);
  const uint8_t *wb = p.w[w_arr] + static_cast<size_t>(u) * CL::kUnitBytes;
  const int grp = u >> p.gs_shift;
  const uint32_t rowb = CL::row_bytes(Tc);
#pragma unroll
  for (int rr = 0; rr < RPT; ++rr) {
    const int r = ph + rr * p.PH;
    if (r < t.nrows) {
      const long long row = r0 + r;
      const uint8_t *src = wb + row * p.row_bytes;
      const uint32_t dst = stage_base + rr * rowb;
#pragma unroll
      for (int c = 0; c < CL::kPlanes; ++c) {
        const uint32_t d = dst + (c * Tc + tid) * CL::kPlane;
        if constexpr (CL::kPlane == 16) cp_async16(d, src + 16 * c);
        else if constexpr (CL::kPlane == 8) cp_async8(d, src + 8 * c);
        else cp_async4(d, src + 4 * c);
      }
      const long long si = row * p.G + grp;
      const uint32_t dsb = dst + Tc * CL::kUnitBytes + tid * 8;
      if (p.sb_pairs) {
        cp_async4(dsb, p.s[w_arr] + (si & ~1LL));
        cp_async4(dsb + 4, p.b[w_arr] + (si & ~1LL));
      }
    }
  }
}

// Read back one row of the thread's unit from ring stage `stage_base`.
template <int BITS>
__device__ __forceinline__ void read_row(const StreamParams &p, uint32_t stage_base,
                                         int rr, int tid, int Tc, int grp_odd,
                                         long long row, int w_arr, int grp,
                                         uint32_t (&w)[BITS], uint32_t &sb) {
  using CL = CopyLayout<BITS>;
  const uint32_t dst = stage_base + rr * CL::row_bytes(Tc);
#pragma unroll
  for (int c = 0; c < CL::kPlanes; ++c) {
    const uint32_t a = dst + (c * Tc + tid) * CL::kPlane;
    if constexpr (CL::kPlane == 16) {
      const uint4 v = lds128(a);
      w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
    } else if constexpr (CL::kPlane == 8) {
      const uint2 v = lds64(a);
      w[2 * c] = v.x; w[2 * c + 1] = v.y;
    } else {
      w[c] = lds32(a);
    }
  }
  if (p.sb_pairs) {
    const uint2 v = lds64(dst + Tc * CL::kUnitBytes + tid * 8);
    // the wanted bf16 is the low half for an even group index, else the high
    const uint32_t s = grp_odd ? (v.x >> 16) : (v.x & 0xffffu);
    const uint32_t b = grp_odd ? (v.y & 0xffff0000u) : (v.y << 16);
    sb = s | b;
  } else {
    const long long si = row * p.G + grp;
    sb = static_cast<uint32_t>(__ldg(p.s[w_arr] + si)) |
         (static_cast<uint32_t>(__ldg(p.b[w_arr] + si)) << 16);
  }
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
        const float send = upper ? vals[i] : vals[i + n / 2];
        const float keep = upper ? vals[i + n / 2] : vals[i];
        vals[i] = keep + __shfl_xor_sync(full, send, off);
      }
      n >>= 1;
    } else {
      vals[0] += __shfl_xor_sync(full, vals[0], off);
    }
  }
}

// The 32 activations of one unit for one activation row (fp32; silu(gate)*up
// in MODE_SILU).  row < 0 marks an absent row (zeros).
__device__ __forceinline__ void unit_activations(const StreamParams &p, int u,
                                                 int row, float (&v)[32]) {
  if (row < 0 || u >= p.U) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = 0.f;
    return;
  }
  const size_t off = static_cast<size_t>(row) * p.K + static_cast<size_t>(u) * 32;
  const uint4 *src = reinterpret_cast<const uint4 *>(p.x + off);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 xv = __ldg(src + q);
    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      v[8 * q + 2 * h] = __uint_as_float(xw[h] << 16);
      v[8 * q + 2 * h + 1] = __uint_as_float(xw[h] & 0xffff0000u);
    }
  }
  if (p.mode == MODE_SILU) {
    // v = silu(gate) * up, kept in fp32
    const uint16_t *up = p.up + off;
#pragma unroll 1
    for (int i = 0; i < 32; ++i) {
      const float g = v[i];
      v[i] = g / (1.0f + expf(-g)) * bf16_to_f32(up[i]);
    }
  }
}

// Per-thread activation state of one unit for MR activation rows.
// Integer path (2/4/8-bit codes): 8-bit digits in the spread layout.
// Float path (3/5/6-bit codes): pre-scaled fp32 activations.
// Both: `back` scales a unit partial back to activation units and
// vs = (sum of the unit's activations) / back, for the bias term.
template <int BITS, int MR>
struct UnitActs {
  static constexpr bool kInt = kIntPath<BITS>;
  int dig[kInt ? MR : 1][3][8];
  float2 xp[kInt ? 1 : MR][16];
  float back[MR], vs[MR];

  __device__ __forceinline__ void load(const StreamParams &p, int u,
                                       const int (&rows)[MR]) {
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      float v[32];
      unit_activations(p, u, rows[m], v);
      if constexpr (kInt) {
        digits_unit<BITS>(v, dig[m], back[m], vs[m]);
      } else {
        float two_c, sum;
        prescale_unit<BITS>(v, xp[m], two_c, sum);
        back[m] = two_c;
        vs[m] = sum * (1.0f / two_c);  // exact: two_c is a power of two
      }
    }
  }
};

// Rows per consumer thread per tile (a compile-time constant per code width).
template <int BITS, int MR, int NSL>
__host__ __device__ constexpr int rows_per_thread() {
  constexpr int base = BITS == 2 ? 16 : (BITS == 3 || BITS == 4) ? 8 : 4;
  return (MR * NSL == 1) ? base : (base / 2 < 2 ? 2 : base / 2);
}

// Partial sums of two rows of the thread's unit: decode, dot products, group
// scale and bias.  Partials stay in the unit's scale; the caller multiplies
// by `back` once per tile.
template <int BITS, int MR>
__device__ __forceinline__ void row_pair_dot(const uint32_t (&w0)[BITS],
                                             uint32_t sb0,
                                             const uint32_t (&w1)[BITS],
                                             uint32_t sb1,
                                             const UnitActs<BITS, MR> &ua,
                                             float *p0, float *p1) {
  float r0[MR], r1[MR];
  if constexpr (kIntPath<BITS>) {
    unit_dp_2rows<BITS, MR>(w0, w1, ua.dig, r0, r1);
  } else {
    float2 a0[MR][2], a1[MR][2];
#pragma unroll
    for (int m = 0; m < MR; ++m)
      a0[m][0] = a0[m][1] = a1[m][0] = a1[m][1] = make_float2(0.f, 0.f);
    unit_fma_2rows<BITS, MR>(w0, w1, ua.xp, a0, a1);
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      const float2 t0 = __fadd2_rn(a0[m][0], a0[m][1]);
      const float2 t1 = __fadd2_rn(a1[m][0], a1[m][1]);
      r0[m] = t0.x + t0.y;
      r1[m] = t1.x + t1.y;
    }
  }
  const float sc0 = __uint_as_float(sb0 << 16);
  const float bi0 = __uint_as_float(sb0 & 0xffff0000u);
  const float sc1 = __uint_as_float(sb1 << 16);
  const float bi1 = __uint_as_float(sb1 & 0xffff0000u);
#pragma unroll
  for (int m = 0; m < MR; ++m) {
    p0[m] = fmaf(bi0, ua.vs[m], fmaf(sc0, r0[m], p0[m]));
    p1[m] = fmaf(bi1, ua.vs[m], fmaf(sc1, r1[m], p1[m]));
  }
}

// BITS: code width; MR: activation rows per segment (1 or 2); NSL: units per
// consumer thread (1 or 2).
template <int BITS, int MR, int NSL>
__global__ void __launch_bounds__(480, 1)
    qmv_stream_kernel(const StreamParams p) {
  constexpr int RPT = rows_per_thread<BITS, MR, NSL>();
  using CL = CopyLayout<BITS>;
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x;
  const int Tc = p.Upad * p.PH / NSL;  // consumer threads
  uint64_t *redfull = reinterpret_cast<uint64_t *>(smem + p.bar_off);
  uint64_t *redempty = redfull + p.nred;

  if (tid == 0) {
    for (int i = 0; i < p.nred; ++i) {
      mbar_init(&redfull[i], Tc / 32);
      mbar_init(&redempty[i], 1);
    }
    fence_mbar_init();
  }
  Groups g{};
  long long V;
  if (p.mode == MODE_GATHER) {
    g = groups_at(smem, p);
    build_groups<MR>(p, g, tid, blockDim.x);  // ends with __syncthreads
    V = static_cast<long long>(*g.nseg) * p.N;
  } else {
    __syncthreads();
    V = static_cast<long long>(p.nmat) * p.nch * p.N;
  }
  const long long v0 = V * blockIdx.x / gridDim.x;
  const long long v1 = V * (blockIdx.x + 1) / gridDim.x;

  if (tid >= Tc) {
    epilogue_loop<MR>(p, smem, redfull, redempty, g, v0, v1, tid - Tc);
    return;
  }

  // ---- consumer set-up: this thread's unit(s) and row phase ----
  const int lane = tid & 31;
  int su[NSL];
#pragma unroll
  for (int j = 0; j < NSL; ++j) su[j] = (tid + j * Tc) % p.Upad;
  const int ph = tid / p.Upad;  // NSL == 2 implies PH == 1 and ph == 0
  const int wslot = su[0] / 32;
  const uint32_t ring = smem_u32(smem) + p.cp_off;
  // one stage = RPT rows for every consumer thread and every slot
  const uint32_t stage_bytes = RPT * NSL * CL::row_bytes(Tc);

  // prefetch: the first depth-1 tiles
  TileWalker tw_issue;
  tw_issue.init(v0, v1, p.N, p.RT, p.depth);
  auto issue_next = [&](int stage) {
    Tile ti;
    if (tw_issue.next(ti)) {
      const Seg si = seg_info<MR>(p, g, ti.seg);
      const int w_arr = p.mode == MODE_GATHER ? 0 : si.arr;
#pragma unroll
      for (int j = 0; j < NSL; ++j)
        if (su[j] < p.U)
          issue_tile<BITS, RPT>(p, ti, si.arr, w_arr, ph, su[j], tid, Tc,
                                ring + stage * stage_bytes +
                                    j * RPT * CL::row_bytes(Tc));
    }
    cp_async_commit();  // possibly empty: keeps the group count regular
  };
  for (int k = 0; k < p.depth - 1; ++k) issue_next(k);

  UnitActs<BITS, MR> ua[NSL];
  int loaded = -1;  // key of the activation rows held in ua

  TileWalker tw;
  tw.init(v0, v1, p.N, p.RT, p.nred);
  Tile t;
  int cstage = 0;
  while (tw.next(t)) {
    const Seg sg = seg_info<MR>(p, g, t.seg);
    if (sg.key != loaded) {
      int xr[MR];
#pragma unroll
      for (int m = 0; m < MR; ++m) xr[m] = seg_xrow<MR>(p, g, sg, m);
#pragma unroll
      for (int j = 0; j < NSL; ++j) ua[j].load(p, su[j], xr);
      loaded = sg.key;
    }
    // keep depth-1 tiles in flight: issue the tile depth-1 ahead, then wait
    // until this tile's copies have landed
    int istage = cstage + p.depth - 1;
    if (istage >= p.depth) istage -= p.depth;
    issue_next(istage);
    switch (p.depth) {  // at most depth-1 newer groups may stay in flight
      case 2: cp_async_wait<1>(); break;
      case 3: cp_async_wait<2>(); break;
      default: cp_async_wait<3>(); break;
    }
    const long long r0 = abs_row(p, sg.arr, t.row);
    const int w_arr = p.mode == MODE_GATHER ? 0 : sg.arr;
    const int nvalid = t.nrows > ph ? min(RPT, (t.nrows - ph + p.PH - 1) / p.PH) : 0;

    float part[RPT * MR];
#pragma unroll
    for (int i = 0; i < RPT * MR; ++i) part[i] = 0.f;
#pragma unroll
    for (int j = 0; j < NSL; ++j) {
      const int u = su[j];
      if (u < p.U) {
        const int grp = u >> p.gs_shift;
        const uint32_t sbase = ring + cstage * stage_bytes + j * RPT * CL::row_bytes(Tc);
        float pj[RPT * MR];
#pragma unroll
        for (int i = 0; i < RPT * MR; ++i) pj[i] = 0.f;
#pragma unroll
        for (int q = 0; q < RPT / 2; ++q) {
          if (2 * q < nvalid) {  // warp-uniform
            uint32_t w0[BITS], w1[BITS], sb0, sb1;
            // a row past the tile end reads the first row's data again
            const int rb1 = 2 * q + 1 < nvalid ? 2 * q + 1 : 2 * q;
            read_row<BITS>(p, sbase, 2 * q, tid, Tc, grp & 1,
                           r0 + ph + 2 * q * p.PH, w_arr, grp, w0, sb0);
            read_row<BITS>(p, sbase, rb1, tid, Tc, grp & 1,
                           r0 + ph + rb1 * p.PH, w_arr, grp, w1, sb1);
            row_pair_dot<BITS, MR>(w0, sb0, w1, sb1, ua[j], pj + (2 * q) * MR,
                                   pj + (2 * q + 1) * MR);
          }
        }
#pragma unroll
        for (int i = 0; i < RPT * MR; ++i)
          part[i] = fmaf(pj[i], ua[j].back[i % MR], part[i]);
      }
    }
    if (++cstage == p.depth) cstage = 0;

    // ---- reduce over the warp's units; one partial per row and x row ----
    const int st = tw.st;
    constexpr int NV = RPT * MR;
    transpose_reduce<NV>(part, lane);
    if (!mbar_wait(&redempty[st], tw.phase ^ 1u)) {
      if (p.err) atomicOr(p.err, 2);
      return;
    }
    float *rbuf = reinterpret_cast<float *>(smem + p.red_off + st * p.red_slot);
    if ((lane % (32 / NV)) == 0) {
      const int idx = lane / (32 / NV);
      const int rr = idx / MR, m = idx % MR;
      const int r = ph + rr * p.PH;
      if (r < t.nrows) rbuf[(r * MR + m) * p.wpr + wslot] = part[0];
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&redfull[st]);
    tw.advance_slot();
  }
  cp_async_wait<0>();  // nothing may be in flight when the thread exits
}

}  // namespace qmvk
