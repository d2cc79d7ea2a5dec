// qmv_stream.cuh -- the persistent weight-streaming GEMV kernel (CUDA cores).
//
// One CTA per SM with three warp roles:
//   * producer warp: streams the weight rows, with their scales and biases,
//     from HBM into a ring of shared-memory slots with 1-D bulk copies that
//     complete on the slot's mbarrier.  A slot holds one or two row pairs of
//     every consumer row phase; the lanes of the warp fill a tile's slots
//     side by side.
//   * consumer warps: each thread owns one 32-code "unit" column of the
//     weight rows (its activations stay in registers) and a row phase.  It
//     decodes its unit of its rows of each slot, multiplies with the
//     activations (8-bit integer dot products for 2/4/8-bit codes, fp32 FMAs
//     for 3/5/6-bit codes), applies the group scale and bias, and the warp
//     reduces the tile's row partials with shuffles into a partial-sum
//     ring slot;
//   * epilogue warp: adds the per-warp partials of each output in a fixed
//     order, adds the residual if any, rounds once to bf16 and stores.
// Slot and partial-sum handoffs are mbarrier phases; consumer warps never
// wait for each other.  Copies move in slots (small, so consumers start soon
// after the first bytes land) while the shuffle reduction and the hand-off
// to the epilogue happen once per tile (many slots).  Tiles are dealt to
// CTAs round-robin, so that at any moment all SMs stream from one compact
// window of memory.
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
// with up to MR activation rows; a segment's N rows are cut into tiles of at
// most RT rows.
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
  int RT;                 // rows per tile (at most RPT * PH)
  int tps;                // tiles per segment: ceil(N / RT)
  int full_slots;         // slots of a full tile: ceil(RT / slot_rows)
  int RA;                 // row alignment making copy starts 16-byte aligned
  int read_once;          // every weight row is streamed once per launch
  int nmat;               // weight matrices (1, or 2 for gate/up)
  int nch;                // activation chunks per matrix: ceil(M / MR)
  int nslot;              // slots in the shared-memory weight ring
  int slot_rows;          // rows per slot: SR rows of every phase (SR * PH)
  int wpr;                // partial-sum slots per row (consumer warps per row)
  uint32_t row_bytes;     // K * bits / 8
  long long total_rows;   // rows in each weight array (N, or E*N)
  int num_pairs, num_x_rows, num_experts;
  uint32_t w_slot, s_slot;    // bytes of a slot's W and S (= B) regions
  uint32_t red_off;           // smem offset of the partial-sum ring
  uint32_t red_stage;         // bytes of one partial-sum ring slot
  int nred;                   // slots in the partial-sum ring
  uint32_t grp_off;           // smem offset of the gather grouping tables
};

// ---------------------------------------------------------------------------
// Tiles.  A segment has tps = ceil(N / RT) tiles; the tiles of all segments
// are numbered segment by segment.  They are dealt to CTAs round-robin (CTA
// c gets tiles c, c + G, c + 2G, ...), so that at any moment all SMs stream
// from one compact window of memory -- or, for the gather mode's many short
// segments, in contiguous blocks (CTA c gets tiles [c*B, (c+1)*B)), so that
// a CTA's consecutive tiles mostly share a segment and its activations.
// Every role of a CTA runs the same walk.
// ---------------------------------------------------------------------------
struct Tile {
  int seg;    // segment index
  int row;    // first row inside the segment's matrix
  int nrows;  // rows in the tile
};

struct TileWalker {
  int seg, tj, tps, nseg, step, N, RT, left;
  int stages, st;
  uint32_t phase;

  __device__ __forceinline__ void init(int nseg_, int N_, int RT_, int tps_,
                                       int stages_, bool blocked = false) {
    N = N_;
    RT = RT_;
    nseg = nseg_;
    stages = stages_;
    tps = tps_;
    st = 0;
    phase = 0;
    if (blocked) {
      const int total = nseg * tps;
      const int B = (total + gridDim.x - 1) / gridDim.x;
      const int start = static_cast<int>(blockIdx.x) * B;
      left = total - start < B ? total - start : B;
      if (left < 0) left = 0;
      step = 1;
      seg = start < total ? start / tps : nseg;
      tj = start < total ? start - seg * tps : 0;
    } else {
      left = 0x7fffffff;
      step = gridDim.x;
      seg = static_cast<int>(blockIdx.x) < tps ? 0 : static_cast<int>(blockIdx.x) / tps;
      tj = blockIdx.x - seg * tps;
    }
  }
  __device__ __forceinline__ bool next(Tile &t) {
    if (seg >= nseg || left <= 0) return false;
    --left;
    t.seg = seg;
    t.row = tj * RT;
    t.nrows = N - t.row < RT ? N - t.row : RT;
    tj += step;
    if (tj >= tps) {
      const int d = tj / tps;
      tj -= d * tps;
      seg += d;
    }
    return true;
  }
  __device__ __forceinline__ void advance_stage() {
    if (++st == stages) {
      st = 0;
      phase ^= 1u;
    }
  }
};

// Position in the slot ring: slot k of the walk is slot k % nslot, in its
// use k / nslot, whose completion is phase parity (k / nslot) & 1.
struct SlotPos {
  int idx;
  uint32_t phase;
  __device__ __forceinline__ SlotPos plus(int n, int nslot) const {
    SlotPos r{idx + n, phase};
    while (r.idx >= nslot) {
      r.idx -= nslot;
      r.phase ^= 1u;
    }
    return r;
  }
};

// Slots of a tile of n rows (a full tile's count is precomputed).
__device__ __forceinline__ int tile_slots(const StreamParams &p, int n) {
  return n == p.RT ? p.full_slots : (n + p.slot_rows - 1) / p.slot_rows;
}

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
__device__ __forceinline__ void build_groups(const StreamParams &p, Groups g, int tid,
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

// One unit (4*BITS bytes, starting at a multiple of 4*BITS) from shared
// memory with the widest aligned loads.
template <int BITS>
__device__ __forceinline__ void lds_unit(uint32_t a, uint32_t (&wd)[BITS]) {
  if constexpr (BITS % 4 == 0) {
#pragma unroll
    for (int i = 0; i < BITS / 4; ++i) {
      const uint4 v = lds128(a + 16 * i);
      wd[4 * i] = v.x; wd[4 * i + 1] = v.y; wd[4 * i + 2] = v.z; wd[4 * i + 3] = v.w;
    }
  } else if constexpr (BITS % 2 == 0) {
#pragma unroll
    for (int i = 0; i < BITS / 2; ++i) {
      const uint2 v = lds64(a + 8 * i);
      wd[2 * i] = v.x; wd[2 * i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < BITS; ++i) wd[i] = lds32(a + 4 * i);
  }
}

// ---------------------------------------------------------------------------
// Producer warp: moves the weight rows with 1-D bulk copies (the copy engine
// does the work; the issuing lanes spend a few instructions per copy).
//
// Slot q of a tile holds tile rows [q*slot_rows, (q+1)*slot_rows) (fewer at
// the tile's end), i.e. SR consecutive rows of every consumer row phase, with
// their scales and biases.  A slot's copy starts at the 16-byte-aligned row
// at or before its first row (`lead` rows earlier).  Lane q fills slot q of
// the tile, so the lanes' waits and address arithmetic run side by side.
//
// bulk_bytes: the bulk part of copying bytes [begin, end) of an array of
// `total` bytes (begin 16-byte aligned).  It ends at a 16-byte boundary:
// rounded up (a few bytes past the slot's rows, never past the array) or,
// at the very end of the array, rounded down; plain_tail copies what
// rounding down left with 2-byte loads and stores.
// ---------------------------------------------------------------------------
constexpr uint32_t kBulkChunk = 16384;  // bytes per bulk copy instruction

__device__ __forceinline__ uint32_t bulk_bytes(long long begin, long long end,
                                               long long total) {
  long long e16 = (end + 15) & ~15LL;
  if (e16 > total) e16 = end & ~15LL;
  return e16 > begin ? static_cast<uint32_t>(e16 - begin) : 0u;
}

__device__ __noinline__ void plain_tail(uint32_t dst, const uint8_t *src,
                                        uint32_t from, uint32_t to) {
  for (uint32_t o = from; o < to; o += 2) {
    const uint16_t v = *reinterpret_cast<const uint16_t *>(src + o);
    asm volatile("st.shared.u16 [%0], %1;\n" ::"r"(dst + o), "h"(v) : "memory");
  }
  // order the plain stores before later bulk writes to this slot
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// When every weight row is streamed once per launch, the weights, scales
// and biases are marked first to go in L2, so the stream does not push out
// what is reused (the kernel's own code, activations, outputs).  Rows read
// again (several chunks of activation rows, or experts revisited by the
// gather mode) keep the normal policy.
__device__ __forceinline__ uint64_t l2_stream_policy(bool read_once) {
  uint64_t pol;
  if (read_once)
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(pol));
  else
    asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;\n" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void bulk_copy(uint32_t dst, const uint8_t *src,
                                          uint32_t bytes, uint64_t *bar, uint64_t pol) {
  for (uint32_t o = 0; o < bytes; o += kBulkChunk) {
    const uint32_t n = bytes - o < kBulkChunk ? bytes - o : kBulkChunk;
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1], %2, [%3], %4;\n" ::"r"(dst + o),
        "l"(src + o), "r"(n), "r"(smem_u32(bar)), "l"(pol)
        : "memory");
  }
}

template <int MR>
__device__ __forceinline__ void producer_loop(const StreamParams &p,
                                              unsigned char *smem, uint64_t *full,
                                              uint64_t *empty, const Groups &g,
                                              int nseg, int lane) {
  TileWalker tw;
  tw.init(nseg, p.N, p.RT, p.tps, 1, p.mode == MODE_GATHER);
  Tile t;
  const uint32_t slot_bytes = p.w_slot + 2 * p.s_slot;
  const uint32_t base = smem_u32(smem);
  const uint32_t rb = p.row_bytes, sb = 2u * p.G;
  const long long wt = p.total_rows * rb, stt = p.total_rows * sb;
  const int q = lane;  // this lane's slot within a tile
  SlotPos pos{0, 0u};
  long long nslots = 0;  // slots filled so far
  bool failed = false;
  bool waited = false;
  while (tw.next(t)) {
    const int ns_t = tile_slots(p, t.nrows);
    const bool active = q < ns_t;
    const SlotPos my = pos.plus(q, p.nslot);
    bool ok = true;
    // a slot's first use needs no wait
    if (active && nslots + q >= p.nslot) ok = mbar_wait(&empty[my.idx], my.phase ^ 1u);
    // warp-uniform outcome: the lanes leave the loop together
    if (!__all_sync(0xffffffffu, ok)) {
      failed = true;
      break;
    }
    uint32_t dw = 0, ds = 0, bw = 0, bs = 0;
    const uint8_t *wsrc = nullptr, *ssrc = nullptr, *bsrc = nullptr;
    if (!waited) {
      grid_dependency_wait();
      waited = true;
    }
    if (active) {
      const Seg sg = seg_info<MR>(p, g, t.seg);
      const int w_arr = p.mode == MODE_GATHER ? 0 : sg.arr;
      const long long a = abs_row(p, sg.arr, t.row) + q * p.slot_rows;
      const int lead = static_cast<int>(a & (p.RA - 1));  // RA: power of two
      const int rows = min(p.slot_rows, t.nrows - q * p.slot_rows);
      const long long a0 = a - lead, a1 = a + rows;
      dw = base + my.idx * slot_bytes;
      ds = dw + p.w_slot;
      wsrc = p.w[w_arr] + a0 * rb;
      ssrc = reinterpret_cast<const uint8_t *>(p.s[w_arr]) + a0 * sb;
      bsrc = reinterpret_cast<const uint8_t *>(p.b[w_arr]) + a0 * sb;
      const uint32_t nw = static_cast<uint32_t>((a1 - a0) * rb);
      const uint32_t ns = static_cast<uint32_t>((a1 - a0) * sb);
      bw = bulk_bytes(a0 * rb, a1 * rb, wt);
      bs = bulk_bytes(a0 * sb, a1 * sb, stt);
      if (bw < nw) plain_tail(dw, wsrc, bw, nw);
      if (bs < ns) {
        plain_tail(ds, ssrc, bs, ns);
        plain_tail(ds + p.s_slot, bsrc, bs, ns);
      }
    }
    if (active) {
      uint64_t *bar = &full[my.idx];
      mbar_arrive_expect_tx(bar, bw + 2 * bs);
      const uint64_t pol = l2_stream_policy(p.read_once != 0);
      bulk_copy(dw, wsrc, bw, bar, pol);
      bulk_copy(ds, ssrc, bs, bar, pol);
      bulk_copy(ds + p.s_slot, bsrc, bs, bar, pol);
    }
    pos = pos.plus(ns_t, p.nslot);
    nslots += ns_t;
  }
  if (failed && p.err && lane == 0) atomicOr(p.err, 2);
  // Before the CTA may exit, every copy the warp started must have landed
  // (consumers normally saw them already): wait for the last use of every
  // slot that was used.
  for (int i = lane; i < p.nslot && i < nslots; i += 32) {
    const long long last = (nslots - 1 - i) / p.nslot;
    mbar_wait(&full[i], static_cast<uint32_t>(last & 1));
  }
}

// ---------------------------------------------------------------------------
// Epilogue warp: sums the consumer warps' partials of each output in a fixed
// order, adds the residual, rounds once to bf16 and stores; then releases the
// partial-sum slot.
// ---------------------------------------------------------------------------
template <int MR>
__device__ __forceinline__ void epilogue_loop(const StreamParams &p,
                                              unsigned char *smem,
                                              uint64_t *redfull,
                                              uint64_t *redempty,
                                              const Groups &g, int nseg,
                                              int lane) {
  grid_dependency_wait();
  TileWalker tw;
  tw.init(nseg, p.N, p.RT, p.tps, p.nred, p.mode == MODE_GATHER);
  Tile t;
  bool dead = false;  // as in the consumers: a wait ran out
  while (tw.next(t)) {
    const int st = tw.st;
    if (!dead && !mbar_wait(&redfull[st], tw.phase)) dead = true;
    const Seg sg = seg_info<MR>(p, g, t.seg);
    const float *rb =
        reinterpret_cast<const float *>(smem + p.red_off + st * p.red_stage);
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
    tw.advance_stage();
  }
  if (dead && p.err) atomicOr(p.err, 2);
}

// ---------------------------------------------------------------------------
// Consumers
// ---------------------------------------------------------------------------

// The raw bf16 words of one unit's activations for one activation row (and,
// in MODE_SILU, of `up`).
struct UnitRaw {
  uint4 x[4], up[4];
  bool valid;
};

template <bool SILU>
__device__ __forceinline__ void fetch_unit(const StreamParams &p, int u, int row,
                                           UnitRaw &r) {
  r.valid = row >= 0 && u < p.U;
  if (!r.valid) return;
  const size_t off = static_cast<size_t>(row) * p.K + static_cast<size_t>(u) * 32;
  const uint4 *src = reinterpret_cast<const uint4 *>(p.x + off);
#pragma unroll
  for (int q = 0; q < 4; ++q) r.x[q] = __ldg(src + q);
  if constexpr (SILU) {
    const uint4 *usrc = reinterpret_cast<const uint4 *>(p.up + off);
#pragma unroll
    for (int q = 0; q < 4; ++q) r.up[q] = __ldg(usrc + q);
  }
}

__device__ __forceinline__ void unpack_bf16x8(const uint4 &w, float *v) {
  const uint32_t xw[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    v[2 * h] = __uint_as_float(xw[h] << 16);
    v[2 * h + 1] = __uint_as_float(xw[h] & 0xffff0000u);
  }
}

// The 32 activations of a fetched unit in fp32: x, or v = silu(gate) * up in
// MODE_SILU (kept in fp32); zeros for an absent row.
template <bool SILU>
__device__ __forceinline__ void unit_values(const UnitRaw &r, float (&v)[32]) {
  if (!r.valid) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = 0.f;
    return;
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) unpack_bf16x8(r.x[q], v + 8 * q);
  if constexpr (SILU) {
    // silu(g) = g / (1 + e^-g) with the fast exponential and division
    // intrinsics (relative error near 2^-21, far inside the tolerance); for
    // g below about -88 the divisor overflows and the result is -0.
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float up[8];
      unpack_bf16x8(r.up[q], up);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float g = v[8 * q + i];
        v[8 * q + i] = __fdividef(g, 1.0f + __expf(-g)) * up[i];
      }
    }
  }
}

// Per-thread activation state of one unit for MR activation rows.
// Integer path (2/4/8-bit codes): 8-bit digits in the spread layout.
// Float path (3/5/6-bit codes): pre-scaled fp32 activations.
// Both: `back` scales a unit partial back to activation units and
// vs = (sum of the unit's activations) / back, for the bias term.
template <int BITS, int MR, bool SILU>
struct UnitActs {
  static constexpr bool kInt = kIntPath<BITS>;
  uint32_t dig[kInt ? MR : 1][3][8];
  float2 xp[kInt ? 1 : MR][16];
  float back[MR], vs[MR];

  __device__ __forceinline__ void load(const StreamParams &p, int u,
                                       const int (&rows)[MR]) {
#pragma unroll
    for (int m = 0; m < MR; ++m) {
      UnitRaw raw;
      fetch_unit<SILU>(p, u, rows[m], raw);
      float v[32];
      unit_values<SILU>(raw, v);
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

// Row pairs per consumer thread in one slot: two, so that the per-slot wait,
// release, address arithmetic and reduction are shared by four rows.
template <int BITS>
__host__ __device__ constexpr int pairs_per_slot() {
  return 2;
}

// Rows per consumer thread per tile: the rows handed to the epilogue at once.
// Eight (four with two units or two activation rows per thread) keeps two
// tiles of the ring within shared memory with up to 16 consumer warps.  The
// gather mode (BIG) keeps taller tiles, 16 rows for codes of up to 4 bits,
// with at most 14 consumer warps: its expert segments are short, and each
// tile pays a reduction and, at a segment change, an activation reload.
template <int BITS, int MR, int NSL, bool BIG = false>
__host__ __device__ constexpr int rows_per_thread() {
  constexpr int base = BIG && (BITS == 2 || BITS == 3 || BITS == 4) ? 16 : 8;
  return (MR * NSL == 1) ? base : base / 2;
}

// Partial sums of two rows of the thread's unit: decode, dot products, group
// scale and bias.  Partials stay in the unit's scale; the caller multiplies
// by `back` once per tile.
template <int BITS, int MR, bool SILU>
__device__ __forceinline__ void row_pair_dot(const uint32_t (&w0)[BITS],
                                             uint32_t sb0,
                                             const uint32_t (&w1)[BITS],
                                             uint32_t sb1,
                                             const UnitActs<BITS, MR, SILU> &ua,
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
// consumer thread (1 or 2); SILU: the activations are silu(gate) * up
// (MODE_SILU only, a separate kernel so the others carry none of its code).
template <int BITS, int MR, int NSL, bool SILU, bool BIG = false>
__global__ void __launch_bounds__(BIG ? 512 : 576, 1)
    qmv_stream_kernel(const StreamParams p) {
  constexpr int RPT = rows_per_thread<BITS, MR, NSL, BIG>();
  extern __shared__ __align__(1024) unsigned char smem[];
  const int tid = threadIdx.x;
  const int Tc = p.Upad * p.PH / NSL;  // consumer threads
  const uint32_t slot_bytes = p.w_slot + 2 * p.s_slot;
  uint64_t *full = reinterpret_cast<uint64_t *>(
      smem + static_cast<size_t>(p.nslot) * slot_bytes);
  uint64_t *empty = full + p.nslot;
  uint64_t *redfull = empty + p.nslot;
  uint64_t *redempty = redfull + p.nred;
  grid_launch_dependents();
  // Each role waits for the previous grid just before its first global
  // access, so that its set-up code runs (and is fetched) while that grid
  // drains; the gather mode reads its index arrays first.

  Groups g{};
  int nseg;
  if (p.mode == MODE_GATHER) {
    grid_dependency_wait();
    g = groups_at(smem, p);
    build_groups<MR>(p, g, tid, blockDim.x);  // ends with __syncthreads
    nseg = *g.nseg;
  } else {
    nseg = p.nmat * p.nch;
  }

  if (tid >= Tc && tid < Tc + 32) {
    // producer warp: its lanes set up the barriers side by side, then it
    // starts streaming at once; the other warps use the barriers only after
    // named barrier 1
    const int lane = tid & 31;
    for (int i = lane; i < p.nslot; i += 32) {
      mbar_init(&full[i], 1);         // the producer lane's expect-tx arrival
      mbar_init(&empty[i], Tc / 32);  // consumer warps
    }
    for (int i = lane; i < p.nred; i += 32) {
      mbar_init(&redfull[i], Tc / 32);
      mbar_init(&redempty[i], 1);     // epilogue warp
    }
    fence_mbar_init();
    __syncwarp();
    named_arrive(1, blockDim.x);
    producer_loop<MR>(p, smem, full, empty, g, nseg, tid & 31);
    return;
  }
  if (tid >= Tc) {
    named_sync(1, blockDim.x);
    epilogue_loop<MR>(p, smem, redfull, redempty, g, nseg, tid & 31);
    return;
  }

  // ---- consumer set-up: this thread's unit(s) and row phase ----
  const int lane = tid & 31;
  int su[NSL];
#pragma unroll
  for (int j = 0; j < NSL; ++j) su[j] = (tid + j * Tc) % p.Upad;
  const int ph = tid / p.Upad;  // NSL == 2 implies PH == 1 and ph == 0
  const int wslot = su[0] / 32;
  const uint32_t row_bytes = p.row_bytes;
  const uint32_t srow_bytes = 2u * p.G;
  const uint32_t rstep = row_bytes * p.PH, sstep = srow_bytes * p.PH;
  const uint32_t smem_base = smem_u32(smem);
  // rows of the thread inside a tile of n rows (warp-uniform)
  auto rows_of = [&](int n) {
    return n > ph ? min(RPT, (n - ph + p.PH - 1) / p.PH) : 0;
  };
  const int nfull = rows_of(p.RT);

  UnitActs<BITS, MR, SILU> ua[NSL];
  int loaded = -1;  // key of the activation rows held in ua

  TileWalker tw;
  tw.init(nseg, p.N, p.RT, p.tps, 1, p.mode == MODE_GATHER);
  // partial-sum ring position of the current tile: slot and phase parity
  int rs = 0;
  uint32_t rphase = 0;

  // The first segment's activations are loaded straight away, while the
  // producer sets up and starts the weight stream, so that these few lines
  // are not queued behind it in HBM.  The mbarriers are used only after
  // named barrier 1, which the producer passes once it has set them up.
  grid_dependency_wait();
  {
    TileWalker w0 = tw;
    Tile t0;
    if (w0.next(t0)) {
      const Seg sg0 = seg_info<MR>(p, g, t0.seg);
      int xr[MR];
#pragma unroll
      for (int m = 0; m < MR; ++m) xr[m] = seg_xrow<MR>(p, g, sg0, m);
#pragma unroll
      for (int j = 0; j < NSL; ++j) ua[j].load(p, su[j], xr);
      loaded = sg0.key;
    }
  }
  named_sync(1, blockDim.x);

  // A wait that runs out marks the thread dead: it records the error and
  // runs to the end without waiting again (results are then garbage), so the
  // warp stays converged for its shuffles.
  bool dead = false;
  auto wait_bar = [&](uint64_t *bar, uint32_t parity) {
    if (!dead && !mbar_wait(bar, parity)) dead = true;
  };

  SlotPos pos{0, 0u};
  Tile t;
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
    const long long ar = abs_row(p, sg.arr, t.row);
    const int nvalid = t.nrows == p.RT ? nfull : rows_of(t.nrows);
    const int ns_t = tile_slots(p, t.nrows);

    // Slot q holds the thread's rows SR*q .. SR*q + SR-1 (SR = 2 * pairs per
    // slot).  For each slot: wait, compute its rows' partials, release it,
    // reduce the partials over the warp's units with a small shuffle
    // butterfly and write them to the tile's partial-sum slot.  The slot
    // loop stays rolled (a compact body stays in the instruction cache).
    // Every warp waits for and releases every slot of the tile, rows or not:
    // a release must not count towards the slot's previous use, which only
    // the refill (after all warps released it) rules out.  Rows past the
    // thread's last row re-read its last row and are dropped at the store.
    constexpr int SPS = pairs_per_slot<BITS>();
    constexpr int SR = 2 * SPS;     // thread rows per slot
    constexpr int NV = SR * MR;     // partials per thread per slot
    wait_bar(&redempty[rs], rphase ^ 1u);
    float *rbuf = reinterpret_cast<float *>(smem + p.red_off + rs * p.red_stage);
#pragma unroll 1
    for (int q = 0; q < ns_t; ++q) {
      const SlotPos my = pos.plus(q, p.nslot);
      wait_bar(&full[my.idx], my.phase);
      const int nv = nvalid - SR * q;  // thread rows in this slot (may be <= 0)
      float part[NV];
#pragma unroll
      for (int i = 0; i < NV; ++i) part[i] = 0.f;
      if (nv > 0) {  // warp-uniform
        const uint32_t lead =
            static_cast<uint32_t>((ar + q * p.slot_rows) & (p.RA - 1));
        const uint32_t sl = smem_base + my.idx * slot_bytes;
        const uint32_t wrow = sl + (lead + ph) * row_bytes;
        const uint32_t srow = sl + p.w_slot + (lead + ph) * srow_bytes;
#pragma unroll
        for (int j = 0; j < NSL; ++j) {
          const int u = su[j];
          if (u < p.U) {
            const uint32_t aw = wrow + static_cast<uint32_t>(u) * (4 * BITS);
            const uint32_t as = srow + 2u * static_cast<uint32_t>(u >> p.gs_shift);
#pragma unroll
            for (int k = 0; k < SPS; ++k) {
              if (2 * k < nv) {  // warp-uniform
                const int ra = 2 * k, rb = 2 * k + 1 < nv ? 2 * k + 1 : 2 * k;
                uint32_t w0[BITS], w1[BITS];
                lds_unit<BITS>(aw + ra * rstep, w0);
                lds_unit<BITS>(aw + rb * rstep, w1);
                const uint32_t sa = as + ra * sstep, sb = as + rb * sstep;
                const uint32_t sb0 = lds16(sa) | (lds16(sa + p.s_slot) << 16);
                const uint32_t sb1 = lds16(sb) | (lds16(sb + p.s_slot) << 16);
                float d0[MR], d1[MR];
#pragma unroll
                for (int m = 0; m < MR; ++m) d0[m] = d1[m] = 0.f;
                row_pair_dot<BITS, MR, SILU>(w0, sb0, w1, sb1, ua[j], d0, d1);
                // back to activation units (per unit)
#pragma unroll
                for (int m = 0; m < MR; ++m) {
                  part[(2 * k) * MR + m] =
                      fmaf(d0[m], ua[j].back[m], part[(2 * k) * MR + m]);
                  part[(2 * k + 1) * MR + m] =
                      fmaf(d1[m], ua[j].back[m], part[(2 * k + 1) * MR + m]);
                }
              }
            }
          }
        }
      }
      // done reading the slot
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[my.idx]);
      // ---- one partial per row and x row over the warp's units ----
      transpose_reduce<NV>(part, lane);
      if ((lane % (32 / NV)) == 0) {
        const int idx = lane / (32 / NV);
        const int rr = idx / MR, m = idx % MR;
        const int r = ph + (SR * q + rr) * p.PH;
        if (rr < nv && r < t.nrows) rbuf[(r * MR + m) * p.wpr + wslot] = part[0];
      }
    }
    pos = pos.plus(ns_t, p.nslot);
    __syncwarp();
    if (lane == 0) mbar_arrive(&redfull[rs]);
    if (++rs == p.nred) {
      rs = 0;
      rphase ^= 1u;
    }
  }
  if (dead && p.err) atomicOr(p.err, 2);
}

}  // namespace qmvk
