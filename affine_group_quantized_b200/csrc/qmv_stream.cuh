// qmv_stream.cuh -- the persistent weight-streaming GEMV kernel (CUDA cores).
//
// One CTA per SM.  The last warp is a producer: one elected lane streams
// tiles of packed weight rows, plus their scales and biases, from HBM into a
// ring of shared-memory stages with 1-D bulk copies (cp.async.bulk) that
// complete on per-stage mbarriers.  The other warps are consumers: each
// thread owns one 32-code "unit" column of the weight rows (its pre-scaled
// activations live in registers), decodes the codes of that unit for several
// rows of the stage, accumulates with packed fp32x2 FMAs, folds in the
// group's scale and bias, and the partial sums are reduced across the row
// with warp shuffles and one shared-memory step.
//
// The same kernel serves every entry point through `mode`:
//   MODE_QMV      y = x @ dequant(W).T
//   MODE_GATE_UP  two weight matrices (gate, up) over one x, one launch
//   MODE_SILU     input v = silu(gate) * up built in fp32; epilogue adds x_resid
//   MODE_GATHER   rows grouped by expert inside the kernel; every touched
//                 expert's rows are streamed once and dotted with all the
//                 x rows routed to it
#pragma once

#include "qmv_device.cuh"

namespace qmvk {

enum Mode : int { MODE_QMV = 0, MODE_GATE_UP = 1, MODE_SILU = 2, MODE_GATHER = 3 };

struct StreamParams {
  const uint8_t *w[2];    // packed rows (segment 0/1); gather: [E*N] rows
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
  int U, Upad;            // units per row (K/32) and padded count
  int PH;                 // row phases: threads per row = Upad, PH rows at once
  int SLOTS;              // units per thread (1 or 2)
  int RPT;                // rows per thread per tile
  int RT;                 // rows per tile = RPT * PH
  int RA;                 // row alignment making copy starts 16-byte aligned
  int nseg;               // 1, or 2 for gate/up
  int stages;
  int wpr;                // reduction slots per row = max(1, Upad / 32)
  long long row_bytes;    // K * bits / 8
  long long total_rows;   // rows in each segment's arrays (N, or E*N)
  int num_pairs, num_x_rows, num_experts;
  uint32_t w_stage, s_stage;  // bytes of W and of S (= B) region per stage
  uint32_t red_off, grp_off;  // smem offsets of reduction / grouping areas
};

// ---------------------------------------------------------------------------
// Tile walk: a CTA owns the virtual rows [v0, v1); tiles never cross a
// segment (matrix or expert) boundary.  Producer and consumers run the same
// walk, so they agree on every tile without communicating.
// ---------------------------------------------------------------------------
struct Tile {
  int seg;       // segment (gate/up matrix, or touched-expert slot)
  int row;       // first row inside the segment
  int nrows;     // rows in the tile
};

__device__ __forceinline__ bool next_tile(long long &v, long long v1, int N,
                                          int RT, Tile &t) {
  if (v >= v1) return false;
  t.seg = static_cast<int>(v / N);
  t.row = static_cast<int>(v - static_cast<long long>(t.seg) * N);
  long long n = RT;
  if (n > N - t.row) n = N - t.row;
  if (n > v1 - v) n = v1 - v;
  t.nrows = static_cast<int>(n);
  v += n;
  return true;
}

// Shared-memory grouping of gather pairs by expert (MODE_GATHER).
struct Groups {
  int *cnt;      // [E]   valid pairs per expert
  int *off;      // [E]   exclusive prefix of cnt
  int *pairs;    // [P]   pair ids, stably ordered by expert
  int *touched;  // [E]   experts with cnt > 0, ascending
  int *ntouched; // [1]
};

__device__ __forceinline__ Groups groups_at(unsigned char *smem,
                                           const StreamParams &p) {
  Groups g;
  int *base = reinterpret_cast<int *>(smem + p.grp_off);
  g.cnt = base;
  g.off = base + p.num_experts;
  g.touched = base + 2 * p.num_experts;
  g.ntouched = base + 3 * p.num_experts;
  g.pairs = base + 3 * p.num_experts + 1;
  return g;
}

// Stable counting sort of the pairs by expert, computed redundantly by every
// CTA (the index arrays are a few hundred bytes).  Pairs with an index out of
// range are dropped and reported through p.status.
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
    // exclusive scan of cnt and the touched list, one warp
    int run = 0, nt = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + tid;
      const int c = e < E ? g.cnt[e] : 0;
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (tid >= o) incl += t;
      }
      if (e < E) g.off[e] = run + incl - c;
      run += __shfl_sync(0xffffffffu, incl, 31);
      const unsigned has = __ballot_sync(0xffffffffu, c > 0);
      if (c > 0) g.touched[nt + __popc(has & ((1u << tid) - 1u))] = e;
      nt += __popc(has);
    }
    if (tid == 0) *g.ntouched = nt;
    __syncwarp();
    // stable scatter: pairs in increasing id order, 32 at a time
    for (int e = tid; e < E; e += 32) g.cnt[e] = 0;  // reuse as cursor
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
      const unsigned same = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(same & ((1u << tid) - 1u));
      const int leader = __ffs(same) - 1;
      int cur = 0;
      if (e >= 0 && tid == leader) cur = g.cnt[e];
      cur = __shfl_sync(0xffffffffu, cur, leader);
      if (e >= 0) g.pairs[g.off[e] + cur + rank] = i;
      __syncwarp();
      if (e >= 0 && tid == leader) g.cnt[e] = cur + __popc(same);
      __syncwarp();
    }
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// Producer: one lane streams tiles into the stage ring.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void copy_rows(unsigned char *dst, const uint8_t *base,
                                         long long row0, long long rows,
                                         long long stride, long long total_rows,
                                         int elem, uint64_t *bar,
                                         uint32_t &tx) {
  // bytes [row0*stride, (row0+rows)*stride) of an array of total_rows rows;
  // row0*stride is 16-byte aligned by construction.
  const long long begin = row0 * stride;
  const long long end = (row0 + rows) * stride;
  const long long total = total_rows * stride;
  long long bulk_end = (end + 15) & ~15LL;
  if (bulk_end > total) bulk_end = end & ~15LL;
  if (bulk_end > begin) {
    const uint32_t nb = static_cast<uint32_t>(bulk_end - begin);
    bulk_g2s(dst, base + begin, nb, bar);
    tx += nb;
  }
  // tail shorter than 16 bytes at the very end of the array: plain copies
  // (elem = 4 for packed words, 2 for bf16), ordered before the barrier
  // arrival by program order.
  for (long long o = bulk_end > begin ? bulk_end : begin; o < end; o += elem) {
    if (elem == 4)
      *reinterpret_cast<uint32_t *>(dst + (o - begin)) =
          *reinterpret_cast<const uint32_t *>(base + o);
    else
      *reinterpret_cast<uint16_t *>(dst + (o - begin)) =
          *reinterpret_cast<const uint16_t *>(base + o);
  }
}

// Row of the tile's first copied row in the segment's arrays, and the
// number of leading rows copied only for alignment.
__device__ __forceinline__ void tile_source(const StreamParams &p, const Tile &t,
                                            const Groups &g, int &seg_arr,
                                            long long &abs_row, int &lead) {
  if (p.mode == MODE_GATHER) {
    seg_arr = 0;
    abs_row = static_cast<long long>(g.touched[t.seg]) * p.N + t.row;
  } else {
    seg_arr = t.seg;
    abs_row = t.row;
  }
  lead = static_cast<int>(abs_row % p.RA);
}

__device__ void producer_loop(const StreamParams &p, unsigned char *smem,
                              uint64_t *full, uint64_t *empty, const Groups &g,
                              long long v0, long long v1) {
  long long v = v0;
  Tile t;
  int it = 0;
  const uint32_t stage_bytes = p.w_stage + 2 * p.s_stage;
  unsigned char *stages = smem;  // stage ring starts at offset 0
  while (next_tile(v, v1, p.N, p.RT, t)) {
    const int st = it % p.stages;
    const uint32_t par = ((it / p.stages) & 1) ^ 1;
    if (!mbar_wait(&empty[st], par)) {
      if (p.err) atomicOr(p.err, 2);
      return;
    }
    int seg_arr, lead;
    long long abs_row;
    tile_source(p, t, g, seg_arr, abs_row, lead);
    unsigned char *dst = stages + static_cast<size_t>(st) * stage_bytes;
    const long long r0 = abs_row - lead;
    const long long nr = lead + t.nrows;
    // Issue the bulk copies and any plain tail stores, then arrive with the
    // byte count: the phase completes once the arrival is in and all bytes
    // have landed, in whichever order those happen.
    uint32_t tx = 0;
    copy_rows(dst, p.w[seg_arr], r0, nr, p.row_bytes, p.total_rows, 4,
              &full[st], tx);
    copy_rows(dst + p.w_stage, reinterpret_cast<const uint8_t *>(p.s[seg_arr]),
              r0, nr, 2LL * p.G, p.total_rows, 2, &full[st], tx);
    copy_rows(dst + p.w_stage + p.s_stage,
              reinterpret_cast<const uint8_t *>(p.b[seg_arr]), r0, nr,
              2LL * p.G, p.total_rows, 2, &full[st], tx);
    mbar_arrive_expect_tx(&full[st], tx);
    ++it;
  }
}

// ---------------------------------------------------------------------------
// Consumers
// ---------------------------------------------------------------------------

// Transposed butterfly: NV partial sums per lane, reduced over L lanes
// (L a power of two <= 32, NV <= L).  Afterwards lane l holds the full sum
// of value index (l % L) / (L / NV) in vals[0].
template <int NV>
__device__ __forceinline__ void transpose_reduce(float (&vals)[NV], int lane,
                                                 int L) {
  int n = NV;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    if (off >= L) continue;
    if (n > 1) {
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int i = 0; i < NV / 2; ++i) {
        if (i < n / 2) {
          const float send = upper ? vals[i] : vals[i + n / 2];
          const float keep = upper ? vals[i + n / 2] : vals[i];
          vals[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      n >>= 1;
    } else {
      vals[0] += __shfl_xor_sync(0xffffffffu, vals[0], off);
    }
  }
}

// Loads the activations a thread needs for one unit and MR x rows, builds
// the pre-scaled registers.  `rows[m]` < 0 marks an absent row (zeros).
template <int BITS, int MR>
__device__ __forceinline__ void load_activations(const StreamParams &p, int u,
                                                 const int (&rows)[MR],
                                                 float2 (&xp)[MR][16],
                                                 float (&two_c)[MR],
                                                 float (&vsum)[MR]) {
#pragma unroll
  for (int m = 0; m < MR; ++m) {
    float v[32];
    if (rows[m] < 0 || u >= p.U) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = 0.f;
    } else {
      const size_t off = static_cast<size_t>(rows[m]) * p.K + static_cast<size_t>(u) * 32;
      const uint4 *src = reinterpret_cast<const uint4 *>(p.x + off);
      if (p.mode == MODE_SILU) {
        const uint4 *usrc = reinterpret_cast<const uint4 *>(p.up + off);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 gv = __ldg(src + q);
          const uint4 uv = __ldg(usrc + q);
          const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
          const uint32_t uw[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const float gg = bf16_to_f32(static_cast<uint16_t>(gw[h] >> (16 * e)));
              const float uu = bf16_to_f32(static_cast<uint16_t>(uw[h] >> (16 * e)));
              v[8 * q + 2 * h + e] = gg / (1.0f + expf(-gg)) * uu;
            }
          }
        }
      } else {
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
      }
    }
    prescale_unit<BITS>(v, xp[m], two_c[m], vsum[m]);
  }
}

// Writes one reduced partial (value index idx = rr * MR + m) of this warp.
template <int MR>
__device__ __forceinline__ void store_partial(float *rb, int idx, int ph, int PH,
                                              int nrows, int wpr, int wslot,
                                              float v) {
  const int rr = idx / MR, m = idx % MR;
  const int r = ph + rr * PH;
  if (r < nrows) rb[(r * MR + m) * wpr + wslot] = v;
}

template <int NV, int MR>
__device__ __forceinline__ void reduce_and_store(const float *part, float *rb,
                                                 int lane, int L, int ph,
                                                 int PH, int nrows, int wpr,
                                                 int wslot) {
  float vals[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) vals[i] = part[i];
  transpose_reduce<NV>(vals, lane, L);
  const int grp_l = L / NV;
  if ((lane % grp_l) == 0)
    store_partial<MR>(rb, (lane % L) / grp_l, ph, PH, nrows, wpr, wslot,
                      vals[0]);
}

// BITS: code width; MR: x rows per pass (1 or 2); NSL: units per thread.
template <int BITS, int MR, int NSL>
__global__ void __launch_bounds__(480, 1)
    qmv_stream_kernel(const StreamParams p) {
  extern __shared__ __align__(128) unsigned char smem[];
  const int tid = threadIdx.x;
  const int Tc = p.Upad * p.PH / NSL;  // consumer threads
  const uint32_t stage_bytes = p.w_stage + 2 * p.s_stage;
  uint64_t *full = reinterpret_cast<uint64_t *>(
      smem + static_cast<size_t>(p.stages) * stage_bytes);
  uint64_t *empty = full + p.stages;
  float *red = reinterpret_cast<float *>(smem + p.red_off);

  if (tid == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], Tc / 32);
    }
    fence_mbar_init();
  }
  Groups g{};
  long long V;
  if (p.mode == MODE_GATHER) {
    g = groups_at(smem, p);
    build_groups(p, g, tid, blockDim.x);  // ends with __syncthreads
    V = static_cast<long long>(*g.ntouched) * p.N;
  } else {
    __syncthreads();
    V = static_cast<long long>(p.nseg) * p.N;
  }
  const long long v0 = V * blockIdx.x / gridDim.x;
  const long long v1 = V * (blockIdx.x + 1) / gridDim.x;

  if (tid >= Tc) {
    if (tid == Tc) producer_loop(p, smem, full, empty, g, v0, v1);
    return;
  }

  // ---- consumer set-up: this thread's unit(s) and row phase ----
  const int lane = tid & 31;
  const int L = p.Upad < 32 ? p.Upad : 32;  // lanes that share a row
  int su[NSL];
#pragma unroll
  for (int j = 0; j < NSL; ++j) su[j] = (tid + j * Tc) % p.Upad;
  const int ph = tid / p.Upad;  // NSL == 2 implies PH == 1 and ph == 0
  const int wslot = p.Upad >= 32 ? su[0] / 32 : 0;

  float2 xp[NSL][MR][16];
  float two_c[NSL][MR], vsum[NSL][MR];
  long long loaded = -1;  // key of the activation rows held in xp
  int rows[MR];

  long long v = v0;
  Tile t;
  int it = 0;
  int rbuf = 0;
  while (next_tile(v, v1, p.N, p.RT, t)) {
    const int st = it % p.stages;
    const uint32_t par = (it / p.stages) & 1;
    int seg_arr, lead;
    long long abs_row;
    tile_source(p, t, g, seg_arr, abs_row, lead);

    int nchunks, gcount = 0, goff = 0;
    if (p.mode == MODE_GATHER) {
      const int e = g.touched[t.seg];
      gcount = g.cnt[e];
      goff = g.off[e];
      nchunks = (gcount + MR - 1) / MR;
    } else {
      nchunks = (p.M + MR - 1) / MR;
    }

    if (!mbar_wait(&full[st], par)) {
      if (p.err) atomicOr(p.err, 2);
      return;
    }
    const unsigned char *sbase = smem + static_cast<size_t>(st) * stage_bytes;
    const uint32_t *wst = reinterpret_cast<const uint32_t *>(sbase);
    const uint16_t *sst = reinterpret_cast<const uint16_t *>(sbase + p.w_stage);
    const uint16_t *bst =
        reinterpret_cast<const uint16_t *>(sbase + p.w_stage + p.s_stage);

    for (int ch = 0; ch < nchunks; ++ch) {
      // activation rows of this chunk; reload only when they change
      const long long key =
          p.mode == MODE_GATHER ? static_cast<long long>(goff + ch * MR) : ch;
      if (key != loaded) {
#pragma unroll
        for (int m = 0; m < MR; ++m) {
          const int i = ch * MR + m;
          if (p.mode == MODE_GATHER) {
            if (i < gcount) {
              const int pr = g.pairs[goff + i];
              rows[m] = p.lhs ? static_cast<int>(p.lhs[pr]) : pr;
            } else {
              rows[m] = -1;
            }
          } else {
            rows[m] = i < p.M ? i : -1;
          }
        }
#pragma unroll
        for (int j = 0; j < NSL; ++j)
          load_activations<BITS, MR>(p, su[j], rows, xp[j], two_c[j], vsum[j]);
        loaded = key;
      }

      float part[MR * 8];
#pragma unroll
      for (int i = 0; i < MR * 8; ++i) part[i] = 0.f;

#pragma unroll
      for (int j = 0; j < NSL; ++j) {
        const int u = su[j];
        if (u < p.U) {
          const int grp = u >> p.gs_shift;
#pragma unroll
          for (int rr = 0; rr < 8; ++rr) {
            const int r = ph + rr * p.PH;
            if (rr < p.RPT && r < t.nrows) {
              const int lr = lead + r;
              uint32_t wd[BITS];
              load_unit<BITS>(
                  wst + (static_cast<size_t>(lr) * p.row_bytes) / 4 +
                      static_cast<size_t>(u) * BITS,
                  wd);
              float2 acc[MR];
#pragma unroll
              for (int m = 0; m < MR; ++m) acc[m] = make_float2(0.f, 0.f);
              unit_fma<BITS, MR>(wd, xp[j], acc);
              const float sc = bf16_to_f32(sst[lr * p.G + grp]);
              const float bi = bf16_to_f32(bst[lr * p.G + grp]);
#pragma unroll
              for (int m = 0; m < MR; ++m) {
                const float R = (acc[m].x + acc[m].y) * two_c[j][m];
                part[rr * MR + m] += fmaf(sc, R, bi * vsum[j][m]);
              }
            }
          }
        }
      }

      // After the last chunk the stage can be refilled: every consumer warp
      // arrives once it is done reading it.
      if (ch == nchunks - 1) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);
      }

      // ---- reduce over the units of each row ----
      float *rb = red + static_cast<size_t>(rbuf) * p.RT * MR * p.wpr;
      switch (p.RPT * MR) {
        case 1: reduce_and_store<1, MR>(part, rb, lane, L, ph, p.PH, t.nrows, p.wpr, wslot); break;
        case 2: reduce_and_store<2, MR>(part, rb, lane, L, ph, p.PH, t.nrows, p.wpr, wslot); break;
        case 4: reduce_and_store<4, MR>(part, rb, lane, L, ph, p.PH, t.nrows, p.wpr, wslot); break;
        case 8: reduce_and_store<8, MR>(part, rb, lane, L, ph, p.PH, t.nrows, p.wpr, wslot); break;
        default:
          if constexpr (MR == 2)
            reduce_and_store<16, MR>(part, rb, lane, L, ph, p.PH, t.nrows, p.wpr, wslot);
          break;
      }
      named_sync(1, Tc);

      // ---- epilogue: one thread per (row, x row) ----
      for (int o = tid; o < t.nrows * MR; o += Tc) {
        const int r = o / MR, m = o % MR;
        float acc = 0.f;
        for (int w = 0; w < p.wpr; ++w) acc += rb[(r * MR + m) * p.wpr + w];
        const int n = t.row + r;
        const int i = ch * MR + m;
        if (p.mode == MODE_GATHER) {
          if (i < gcount) {
            const int pr = g.pairs[goff + i];
            p.y[0][static_cast<size_t>(pr) * p.N + n] = f32_to_bf16(acc);
          }
        } else if (i < p.M) {
          const size_t yo = static_cast<size_t>(i) * p.N + n;
          if (p.mode == MODE_SILU && p.resid) acc += bf16_to_f32(p.resid[yo]);
          p.y[seg_arr][yo] = f32_to_bf16(acc);
        }
      }
      rbuf ^= 1;
    }
    ++it;
  }
}

}  // namespace qmvk
