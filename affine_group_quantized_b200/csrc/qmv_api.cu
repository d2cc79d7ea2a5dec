// qmv_api.cu -- the C ABI of libqmv: argument checks, launch planning and
// kernel dispatch.  Declarations and the contract of every entry point are in
// include/qmv.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>

#include <cuda_fp16.h>

#include "qmv.h"
#include "qmv_decode.cuh"
#include "qmv_mma.cuh"
#include "qmv_qmm.h"
#include "qmv_qvm.cuh"
#include "qmv_stream.cuh"
#include "qmv_trellis.cuh"

namespace {

thread_local std::string g_last_error;

int fail(int code, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int ok() {
  g_last_error.clear();
  return QMV_OK;
}

// Launch with programmatic stream serialization allowed: the kernel may be
// scheduled while the previous kernel on the stream is finishing; it holds
// its first global access until that kernel has completed (the kernels
// start with griddepcontrol.wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), int grid, int threads, int smem,
                       cudaStream_t stream, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

bool aligned16(const void *p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

bool bits_supported(int bits) {
  return bits == 2 || bits == 3 || bits == 4 || bits == 5 || bits == 6 ||
         bits == 8;
}

bool gs_supported(int gs) { return gs == 32 || gs == 64 || gs == 128; }

int gcd_i(int a, int b) {
  while (b) {
    const int t = a % b;
    a = b;
    b = t;
  }
  return a;
}

// Status word of the GEMV kernels, one per device: a kernel ORs 2 into it
// when one of its bounded waits gives up (that launch's results are then
// undefined).  Read and cleared with qmv_device_status.
static __device__ int g_device_status;

// Per-device facts, queried once per device.
struct DeviceInfo {
  int sms = 0;
  int smem_optin = 0;
  int *status = nullptr;        // device address of g_device_status
  cudaError_t status_err = cudaSuccess;
};
constexpr int kMaxDevices = 64;
#ifndef QMV_MMA_MIN_ROWS
#define QMV_MMA_MIN_ROWS 3
#endif
// fewest activation rows that go to the tensor-core path
constexpr int kMmaMinRows = QMV_MMA_MIN_ROWS;
#ifndef QMV_QMM_MIN_ROWS
#define QMV_QMM_MIN_ROWS 17
#endif
// fewest activation rows that go to the many-row tensor-core kernel
constexpr int kQmmMinRows = QMV_QMM_MIN_ROWS;
DeviceInfo g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];

int device_info(DeviceInfo **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return fail(QMV_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return fail(QMV_ERR_CUDA, "device index %d out of range", dev);
  int rc = QMV_OK;
  std::call_once(g_dev_once[dev], [&] {
    cudaError_t e1 = cudaDeviceGetAttribute(&g_dev[dev].sms,
                                            cudaDevAttrMultiProcessorCount, dev);
    cudaError_t e2 = cudaDeviceGetAttribute(
        &g_dev[dev].smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e1 != cudaSuccess || e2 != cudaSuccess) g_dev[dev].sms = 0;
    // the status word's device address, with this device current
    void *a = nullptr;
    g_dev[dev].status_err = cudaGetSymbolAddress(&a, g_device_status);
    if (g_dev[dev].status_err == cudaSuccess) g_dev[dev].status = static_cast<int *>(a);
  });
  if (g_dev[dev].sms <= 0)
    return fail(QMV_ERR_CUDA, "cannot query device %d attributes", dev);
  if (!g_dev[dev].status)
    return fail(QMV_ERR_CUDA, "cudaGetSymbolAddress(status word): %s",
                cudaGetErrorString(g_dev[dev].status_err));
  *out = &g_dev[dev];
  return rc;
}

// Common shape checks of the pages' shape rule: w holds K*bits/32 words per
// row and K/group_size groups (extract_quantized_matmul_dims).
int check_common(int N, int K, int bits, int gs) {
  if (!bits_supported(bits))
    return fail(QMV_ERR_UNSUPPORTED, "bits=%d not in {2,3,4,5,6,8}", bits);
  if (!gs_supported(gs))
    return fail(QMV_ERR_UNSUPPORTED, "group_size=%d not in {32,64,128}", gs);
  if (N <= 0) return fail(QMV_ERR_SHAPE, "N=%d must be positive", N);
  if (K <= 0) return fail(QMV_ERR_SHAPE, "K=%d must be positive", K);
  if (K % gs != 0)
    return fail(QMV_ERR_SHAPE, "K=%d is not a multiple of group_size=%d", K, gs);
  if (K > 28672)
    return fail(QMV_ERR_UNSUPPORTED, "K=%d above the supported 28672", K);
  return QMV_OK;
}

// ---------------------------------------------------------------------------
// Launch planning for the streaming kernel
// ---------------------------------------------------------------------------
struct Plan {
  qmvk::StreamParams p;
  int mr = 1, nsl = 1;
  bool big = false;  // taller tiles (gather mode)
  int threads = 0;
  size_t smem = 0;
  int grid = 0;
};

// Rows per consumer thread per tile; the same rule as the kernel's
// rows_per_thread<BITS, MR, NSL, BIG>() (BIG: the gather mode).
int rows_per_thread_host(int bits, int mr, int nsl, bool big) {
  const int base = big && (bits == 2 || bits == 3 || bits == 4) ? 16 : 8;
  return (mr * nsl == 1) ? base : base / 2;
}

// Thread layout: Upad (>= 32, a multiple of 32) consumer threads cover the
// 32-code units of one row, PH such groups work on PH rows at once; each
// consumer thread handles up to RPT rows of its unit per tile.  A producer
// warp and an epilogue warp complete the CTA.  Stages hold RT rows (plus the
// rows copied only for alignment) of weights, scales and biases.
int make_plan(Plan &pl, int bits, int gs, int mr_want, DeviceInfo *dev) {
  qmvk::StreamParams &p = pl.p;
  const int K = p.K;
  const int U = K / 32;
  int Upad = U < 32 ? 32 : (U + 31) / 32 * 32;
  int nsl = 1;
  if (Upad > 448) {
    Upad = (U + 63) / 64 * 64;
    nsl = 2;
  }
  const int mr = (nsl == 1 && mr_want >= 2) ? 2 : 1;
  const long long row_bytes = static_cast<long long>(K) * bits / 8;
  const int G = K / gs;
  const bool big = p.mode == qmvk::MODE_GATHER;
  const int RPT = rows_per_thread_host(bits, mr, nsl, big);
  long long grp_bytes = 0;
  if (p.mode == qmvk::MODE_GATHER)
    grp_bytes = (2LL * p.num_experts + 3LL * p.num_pairs + 1) * 4;
  const int ra_w = 16 / gcd_i(static_cast<int>(row_bytes % 16 == 0 ? 16 : row_bytes % 16), 16);
  const int ra_s = 16 / gcd_i((2 * G) % 16 == 0 ? 16 : (2 * G) % 16, 16);
  const int RA = ra_w * ra_s / gcd_i(ra_w, ra_s);
  const int wpr = Upad / 32 / nsl;
  // consumer threads: up to 512 (plus producer and epilogue warps: 576 per
  // CTA, at most 113 registers per thread).  A slot holds SR rows of every row
  // phase (SR = 2 * pairs per slot, the kernel's pairs_per_slot<BITS>); the
  // ring must hold the slots of two tiles (RPT / SR each), so the row phases
  // are reduced until it does.
  const int SR = 2 * 2;  // the kernel's 2 * pairs_per_slot<BITS>()
  const int tc_max = big ? 448 : 512;
  int PH = nsl == 1 && Upad <= tc_max ? tc_max / Upad : 1;
  struct Sizes { long long w, s, red, slot; };
  auto sizes = [&](int ph) {
    Sizes z;
    const long long rows = static_cast<long long>(SR) * ph + RA - 1;
    z.w = (rows * row_bytes + 16 + 15) / 16 * 16;
    z.s = (rows * 2LL * G + 16 + 15) / 16 * 16;
    z.red = (static_cast<long long>(RPT) * ph * mr * wpr * 4 + 15) / 16 * 16;
    z.slot = z.w + 2 * z.s;
    return z;
  };
  const int nred = 4;
  auto slots_of = [&](int ph) {
    const Sizes z = sizes(ph);
    return (dev->smem_optin - grp_bytes - 256 - nred * (z.red + 16)) / (z.slot + 16);
  };
  const int tile_slots_max = (RPT + SR - 1) / SR;
  while (PH > 1 && slots_of(PH) < 2 * tile_slots_max) --PH;
  const int Tc = Upad * PH / nsl;
  if (Tc > tc_max || Tc % 32 != 0)
    return fail(QMV_ERR_UNSUPPORTED, "K=%d has no thread layout", K);
  const Sizes z = sizes(PH);
  long long ns = slots_of(PH);
  if (ns > 32) ns = 32;
  if (ns < tile_slots_max)
    return fail(QMV_ERR_UNSUPPORTED, "shape needs more shared memory than the device offers");
  const int RT = RPT * PH;
  p.gs_shift = 0;
  while ((32 << p.gs_shift) < gs) ++p.gs_shift;
  p.G = G;
  p.U = U;
  p.Upad = Upad;
  p.PH = PH;
  p.RT = RT;
  p.RA = RA;
  p.nslot = static_cast<int>(ns);
  p.slot_rows = SR * PH;
  p.wpr = wpr;
  p.row_bytes = static_cast<uint32_t>(row_bytes);
  p.nch = p.mode == qmvk::MODE_GATHER ? 1 : (p.M + mr - 1) / mr;
  p.read_once = p.mode != qmvk::MODE_GATHER && p.nch == 1;
  p.w_slot = static_cast<uint32_t>(z.w);
  p.s_slot = static_cast<uint32_t>(z.s);
  const long long ring = ns * z.slot;
  p.red_off = static_cast<uint32_t>((ring + (2 * ns + 2 * nred) * 8 + 15) / 16 * 16);
  p.red_stage = static_cast<uint32_t>(z.red);
  p.nred = nred;
  p.grp_off = static_cast<uint32_t>(p.red_off + nred * z.red);
  pl.smem = static_cast<size_t>(p.grp_off + grp_bytes);
  pl.mr = mr;
  pl.nsl = nsl;
  pl.big = big;
  pl.threads = Tc + 64;
  // One CTA per SM (fewer when there are fewer tiles).  Tiles are dealt
  // round-robin, so the tile height is lowered until every CTA gets the
  // same number of tiles to within one.
  long long grid = dev->sms;
  if (p.mode != qmvk::MODE_GATHER) {
    const long long nseg = static_cast<long long>(p.nmat) * p.nch;
    if (nseg * p.N > 0x7fffffffLL)
      return fail(QMV_ERR_UNSUPPORTED, "too many output rows in one call");
    const long long tiles = nseg * ((p.N + RT - 1) / RT);
    if (tiles < grid) grid = tiles;
    const long long per_cta = (tiles + grid - 1) / grid;
    const long long tps_want = (per_cta * grid + nseg - 1) / nseg;
    long long rte = (p.N + tps_want - 1) / tps_want;
    if (rte < 1) rte = 1;
    if (rte > RT) rte = RT;
    p.RT = static_cast<int>(rte);
  }
  pl.grid = static_cast<int>(grid < 1 ? 1 : grid);
  // walk constants for the final tile height
  p.tps = (p.N + p.RT - 1) / p.RT;
  p.full_slots = (p.RT + p.slot_rows - 1) / p.slot_rows;
  return QMV_OK;
}

template <int BITS, int MR, int NSL, bool SILU, bool BIG>
int &granted_smem(int dev) {
  static int granted[kMaxDevices] = {};
  return granted[dev];
}

template <int BITS, int MR, int NSL, bool SILU, bool BIG = false>
int launch_t(const Plan &pl, cudaStream_t stream) {
  auto kern = qmvk::qmv_stream_kernel<BITS, MR, NSL, SILU, BIG>;
  int dev = 0;
  cudaGetDevice(&dev);
  int &granted = granted_smem<BITS, MR, NSL, SILU, BIG>(dev);
  if (static_cast<int>(pl.smem) > granted) {
    cudaError_t e = cudaFuncSetAttribute(
        kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
        static_cast<int>(pl.smem));
    if (e != cudaSuccess)
      return fail(QMV_ERR_CUDA, "cudaFuncSetAttribute: %s",
                  cudaGetErrorString(e));
    granted = static_cast<int>(pl.smem);
  }
  const cudaError_t le = launch_pdl(kern, pl.grid, pl.threads, pl.smem, stream, pl.p);
  if (le != cudaSuccess) {
    cudaGetLastError();  // clear it
    return fail(QMV_ERR_CUDA, "kernel launch: %s", cudaGetErrorString(le));
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(QMV_ERR_CUDA, "kernel launch: %s", cudaGetErrorString(e));
  return ok();
}

template <int BITS, bool SILU>
int launch_shape(const Plan &pl, cudaStream_t stream) {
  if constexpr (!SILU) {
    if (pl.big) {  // gather mode: taller tiles
      if (pl.nsl == 2) return launch_t<BITS, 1, 2, false, true>(pl, stream);
      if (pl.mr == 2) return launch_t<BITS, 2, 1, false, true>(pl, stream);
      return launch_t<BITS, 1, 1, false, true>(pl, stream);
    }
  }
  if (pl.nsl == 2) return launch_t<BITS, 1, 2, SILU>(pl, stream);
  if (pl.mr == 2) return launch_t<BITS, 2, 1, SILU>(pl, stream);
  return launch_t<BITS, 1, 1, SILU>(pl, stream);
}

template <int BITS>
int launch_bits(const Plan &pl, cudaStream_t stream) {
  if (pl.p.mode == qmvk::MODE_SILU) return launch_shape<BITS, true>(pl, stream);
  return launch_shape<BITS, false>(pl, stream);
}

int launch(const Plan &pl, int bits, cudaStream_t stream) {
  switch (bits) {
    case 2: return launch_bits<2>(pl, stream);
    case 3: return launch_bits<3>(pl, stream);
    case 4: return launch_bits<4>(pl, stream);
    case 5: return launch_bits<5>(pl, stream);
    case 6: return launch_bits<6>(pl, stream);
    case 8: return launch_bits<8>(pl, stream);
    default: return fail(QMV_ERR_UNSUPPORTED, "bits=%d", bits);
  }
}

void init_params(qmvk::StreamParams &p) { std::memset(&p, 0, sizeof p); }

// ---------------------------------------------------------------------------
// The decode kernel (qmv_decode.cuh): one activation row, 2- or 4-bit codes,
// rows of a multiple of 2048 codes.  Other shapes take the streaming kernel.
// ---------------------------------------------------------------------------

// The decode kernel takes 2- and 4-bit codes, where the streaming kernel's
// per-code work was the limit; for 3-, 5-, 6- and 8-bit codes the streaming
// kernel measured as fast or faster.
bool decode_path(int M, int K, int bits) {
  return M == 1 && (bits == 2 || bits == 4) && K % 2048 == 0 && K <= 28672;
}

struct DecodePlan {
  qmvk::DecodeParams p;
  int grid = 0, threads = 0;
  size_t smem = 0;
};

// Consumer warps: the most whole rows of warps (K / 2048 warps per row)
// within kDecodeMaxWarps; slots of decode_rps<BITS>() rows per row phase; as many
// slots as fit next to the partial sums, the span records, the activations
// and the barriers.  Returns false when not even two slots fit (the caller
// then takes the streaming kernel).
bool make_decode_plan(DecodePlan &dp, int bits, int gs, bool silu, DeviceInfo *dev) {
  qmvk::DecodeParams &p = dp.p;
  const int K = p.K;
  const int rps = qmvk::kDecodeRps;
  const int rec_words = qmvk::kSpanRec;
  p.WPR = K / 2048;
  p.G = K / gs;
  p.row_bytes = static_cast<uint32_t>(static_cast<long long>(K) * bits / 8);
  const long long dig = static_cast<long long>(K / qmvk::kSpan) * rec_words * 4;
  const long long xs = (silu ? 4LL : 2LL) * K;
  // the most row phases whose ring still holds three slots (two if even one
  // row phase does not)
  int best_ph = 0, best_ns = 0;
  for (int ph = qmvk::kDecodeMaxWarps / p.WPR; ph >= 1; --ph) {
    const int SR = ph * rps;
    const long long slot_w = static_cast<long long>(SR) * p.row_bytes;
    const long long slot_s = static_cast<long long>(SR) * 2 * p.G;
    const long long slot_bytes = (slot_w + 2 * slot_s + 127) / 128 * 128;
    int ns = 0;
    for (int k = 32; k >= 2; --k) {
      const long long part = (static_cast<long long>(k) * 2 * SR * p.WPR * 4 + 15) / 16 * 16;
      if (static_cast<long long>(k) * slot_bytes + part + dig + xs + 2LL * k * 8 <=
          dev->smem_optin) {
        ns = k;
        break;
      }
    }
    if (ns >= 3 || (ns >= 2 && ph == 1)) {
      best_ph = ph;
      best_ns = ns;
      break;
    }
  }
  if (best_ns < 2) return false;
  p.PH = best_ph;
  p.SR = p.PH * rps;
  p.slot_w = static_cast<uint32_t>(p.SR) * p.row_bytes;
  p.slot_s = static_cast<uint32_t>(p.SR) * 2u * static_cast<uint32_t>(p.G);
  p.slot_bytes = (p.slot_w + 2 * p.slot_s + 127) / 128 * 128;
  p.nslot = best_ns;
  const long long part = (static_cast<long long>(p.nslot) * 2 * p.SR * p.WPR * 4 + 15) / 16 * 16;
  p.part_off = static_cast<uint32_t>(static_cast<long long>(p.nslot) * p.slot_bytes);
  p.dig_off = static_cast<uint32_t>(p.part_off + part);
  p.x_off = static_cast<uint32_t>(p.dig_off + dig);
  p.bar_off = static_cast<uint32_t>(p.x_off + xs);
  dp.smem = static_cast<size_t>(p.bar_off) + 2u * p.nslot * 8;
  long long grid = dev->sms;
  if (p.total_rows < grid) grid = p.total_rows;
  dp.grid = static_cast<int>(grid);
  dp.threads = (p.WPR * p.PH + 1) * 32;
  return true;
}

template <int BITS, int GS, bool SILU>
int launch_decode_t(const DecodePlan &dp, cudaStream_t stream) {
  auto kern = qmvk::qmv_decode_kernel<BITS, GS, SILU>;
  int dev = 0;
  cudaGetDevice(&dev);
  static int granted[kMaxDevices] = {};
  if (static_cast<int>(dp.smem) > granted[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(dp.smem));
    if (e != cudaSuccess)
      return fail(QMV_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    granted[dev] = static_cast<int>(dp.smem);
  }
  const cudaError_t le = launch_pdl(kern, dp.grid, dp.threads, static_cast<int>(dp.smem),
                                    stream, dp.p);
  if (le != cudaSuccess) {
    cudaGetLastError();  // clear it
    return fail(QMV_ERR_CUDA, "kernel launch: %s", cudaGetErrorString(le));
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(QMV_ERR_CUDA, "kernel launch: %s", cudaGetErrorString(e));
  return ok();
}

template <int BITS, bool SILU>
int launch_decode_b(const DecodePlan &dp, int gs, cudaStream_t stream) {
  switch (gs) {
    case 32: return launch_decode_t<BITS, 32, SILU>(dp, stream);
    case 64: return launch_decode_t<BITS, 64, SILU>(dp, stream);
    case 128: return launch_decode_t<BITS, 128, SILU>(dp, stream);
    default: return fail(QMV_ERR_UNSUPPORTED, "group_size=%d", gs);
  }
}

template <bool SILU>
int launch_decode(const DecodePlan &dp, int bits, int gs, cudaStream_t stream) {
  switch (bits) {
    case 2: return launch_decode_b<2, SILU>(dp, gs, stream);
    case 4: return launch_decode_b<4, SILU>(dp, gs, stream);
    default: return fail(QMV_ERR_UNSUPPORTED, "bits=%d on the decode kernel", bits);
  }
}

// Fills the matrix-independent fields of a decode plan.
void init_decode(DecodePlan &dp, const void *x, int N, int K, int nmat, const DeviceInfo *dev) {
  std::memset(&dp.p, 0, sizeof dp.p);
  dp.p.err = dev->status;
  dp.p.x = static_cast<const uint16_t *>(x);
  dp.p.N = N;
  dp.p.K = K;
  dp.p.total_rows = static_cast<long long>(nmat) * N;
}

// ---------------------------------------------------------------------------
// Batched rows on the tensor cores (qmv_mma.cuh): up to 16 activation rows
// share one read of the weights.  2-, 4- and 8-bit codes; K a multiple of
// one stage row (1024 / bits codes); group sizes 32, 64, 128.
// ---------------------------------------------------------------------------
// (K / gs) % 8 == 0 makes the scale / bias row stride a multiple of 16 bytes
// (a tensor-copy rule).
bool mma_path(int M, int K, int bits, int gs) {
  if (!(bits == 2 || bits == 4 || bits == 8)) return false;
  if (!(gs == 32 || gs == 64 || gs == 128)) return false;
  return M >= kMmaMinRows && M <= qmvk::kMmaCols && M < kQmmMinRows &&
         K % (1024 / bits) == 0 && (K / gs) % 8 == 0;
}

// cuTensorMapEncodeTiled, looked up once through the runtime (no link to
// the driver library).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// A 2-D row-major tensor [rows][cols] of `esize`-byte elements with row
// stride `stride` bytes, copied in boxes of [box_rows][box_cols].
int encode_2d(CUtensorMap *map, const void *ptr, CUtensorMapDataType type, uint64_t cols,
              uint64_t rows, uint64_t stride, uint32_t box_cols, uint32_t box_rows,
              CUtensorMapSwizzle swz, CUtensorMapL2promotion l2) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return fail(QMV_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {stride};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, type, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, swz, l2,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(QMV_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return 0;
}

// Scratch of the tensor-core path, one per device, made on first use and
// grown when a call needs more: the partial-sum slots (two per CTA) and one
// arrival counter per tile (zero between launches: the last arrival resets
// it).  Calls that use it on one device are expected in stream order.
struct MmaScratch {
  float *part = nullptr;
  size_t part_bytes = 0;
  int *cnt = nullptr;
  int cnt_len = 0;
};
MmaScratch g_mma_scratch[kMaxDevices];
std::mutex g_mma_scratch_mu;

int mma_scratch(int dev_id, size_t part_bytes, int ntiles, cudaStream_t stream,
                MmaScratch **out) {
  std::lock_guard<std::mutex> lock(g_mma_scratch_mu);
  MmaScratch &s = g_mma_scratch[dev_id];
  if (s.part_bytes < part_bytes) {
    float *np = nullptr;
    if (cudaMalloc(&np, part_bytes) != cudaSuccess)
      return fail(QMV_ERR_CUDA, "tensor-core path: cannot allocate %zu bytes of scratch",
                  part_bytes);
    if (s.part) cudaFree(s.part);  // waits for the launches that use it
    s.part = np;
    s.part_bytes = part_bytes;
  }
  if (s.cnt_len < ntiles) {
    int n = s.cnt_len ? s.cnt_len : 1024;
    while (n < ntiles) n *= 2;
    int *c = nullptr;
    // zeroed on the caller's stream, so the launch that follows on that
    // stream sees the zeros whatever kind of stream it is
    if (cudaMalloc(&c, static_cast<size_t>(n) * 4) != cudaSuccess)
      return fail(QMV_ERR_CUDA, "tensor-core path: cannot allocate the tile counters");
    if (cudaMemsetAsync(c, 0, static_cast<size_t>(n) * 4, stream) != cudaSuccess) {
      cudaFree(c);
      return fail(QMV_ERR_CUDA, "tensor-core path: cannot clear the tile counters");
    }
    if (s.cnt) cudaFree(s.cnt);  // waits for the launches that use it
    s.cnt = c;
    s.cnt_len = n;
  }
  *out = &s;
  return 0;
}

// The same scratch for qmv_noalloc, as a fixed array in the library's device
// image: partial-sum slots for up to kStaticCtas CTAs, then arrival counters
// for up to kStaticTiles tiles (zero at load; every launch leaves them zero).
constexpr int kStaticCtas = 256;
constexpr int kStaticTiles = 1 << 16;
constexpr size_t kStaticPartBytes =
    static_cast<size_t>(kStaticCtas) * 2 * qmvk::kMmaCols * qmvk::kMmaRows * 4;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticPartBytes +
                                                                 kStaticTiles * 4];
MmaScratch g_static_view[kMaxDevices];
cudaError_t g_static_err[kMaxDevices];
std::once_flag g_static_once[kMaxDevices];

int static_scratch(int dev_id, int sms, int ntiles, MmaScratch **out) {
  if (sms > kStaticCtas || ntiles > kStaticTiles)
    return fail(QMV_ERR_UNSUPPORTED,
                "qmv_noalloc: %d SMs / %d row tiles exceed the fixed scratch (%d / %d)", sms,
                ntiles, kStaticCtas, kStaticTiles);
  std::call_once(g_static_once[dev_id], [&] {
    void *a = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&a, g_static_scratch);
    g_static_err[dev_id] = e;
    if (e == cudaSuccess) {
      g_static_view[dev_id].part = static_cast<float *>(a);
      g_static_view[dev_id].cnt = reinterpret_cast<int *>(static_cast<unsigned char *>(a) +
                                                          kStaticPartBytes);
      g_static_view[dev_id].cnt_len = kStaticTiles;
    }
  });
  if (!g_static_view[dev_id].part)
    return fail(QMV_ERR_CUDA, "qmv_noalloc: cudaGetSymbolAddress: %s",
                cudaGetErrorString(g_static_err[dev_id]));
  *out = &g_static_view[dev_id];
  return 0;
}

template <int BITS, int GS>
int launch_mma_t(qmvk::MmaParams &mp, int grid, DeviceInfo *dev, cudaStream_t stream) {
  using ST = qmvk::MmaStage<BITS>;
  auto kern = qmvk::qmv_mma_kernel<BITS, GS>;
  mp.stage_bytes = ST::bytes(mp.M);
  const int room = dev->smem_optin - static_cast<int>(qmvk::MmaSmem::w_off) - 1024;
  int nst = room / static_cast<int>(mp.stage_bytes);
  if (nst > qmvk::kMmaMaxStages) nst = qmvk::kMmaMaxStages;
  if (nst < 2) return fail(QMV_ERR_UNSUPPORTED, "tensor-core path: shared memory too small");
  mp.nst = nst;
  const int smem = static_cast<int>(qmvk::MmaSmem::w_off + 1024 + nst * mp.stage_bytes);
  // tensor maps: codes [N][row_bytes] u8, scales / biases [N][G] u16,
  // x [M][K] u16
  CUtensorMap tw, ts, tb, tx;
  int rc;
  if ((rc = encode_2d(&tw, mp.w, CU_TENSOR_MAP_DATA_TYPE_UINT8, mp.row_bytes, mp.N, mp.row_bytes,
                      128, qmvk::kMmaRows, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B)))
    return rc;
  if ((rc = encode_2d(&ts, mp.s, CU_TENSOR_MAP_DATA_TYPE_UINT16, mp.G, mp.N, 2ull * mp.G,
                      qmvk::kMmaWinGroups, qmvk::kMmaRows, CU_TENSOR_MAP_SWIZZLE_32B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_128B)))
    return rc;
  if ((rc = encode_2d(&tb, mp.b, CU_TENSOR_MAP_DATA_TYPE_UINT16, mp.G, mp.N, 2ull * mp.G,
                      qmvk::kMmaWinGroups, qmvk::kMmaRows, CU_TENSOR_MAP_SWIZZLE_32B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_128B)))
    return rc;
  if ((rc = encode_2d(&tx, mp.x, CU_TENSOR_MAP_DATA_TYPE_UINT16, mp.K, mp.M, 2ull * mp.K,
                      qmvk::mma_x_slice<BITS>(), mp.M, CU_TENSOR_MAP_SWIZZLE_NONE,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_128B)))
    return rc;
  int d = 0;
  cudaGetDevice(&d);
  static int granted[kMaxDevices] = {};
  if (smem > granted[d]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         dev->smem_optin);
    if (e != cudaSuccess)
      return fail(QMV_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    granted[d] = dev->smem_optin;
  }
  const cudaError_t le =
      launch_pdl(kern, grid, qmvk::mma_threads<BITS>(), smem, stream, tw, ts, tb, tx, mp);
  if (le != cudaSuccess) {
    cudaGetLastError();  // clear it
    return fail(QMV_ERR_CUDA, "kernel launch: %s", cudaGetErrorString(le));
  }
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return fail(QMV_ERR_CUDA, "kernel launch: %s", cudaGetErrorString(e));
  return ok();
}

template <int BITS>
int launch_mma_b(qmvk::MmaParams &mp, int gs, int grid, DeviceInfo *dev, cudaStream_t stream) {
  switch (gs) {
    case 32: return launch_mma_t<BITS, 32>(mp, grid, dev, stream);
    case 64: return launch_mma_t<BITS, 64>(mp, grid, dev, stream);
    case 128: return launch_mma_t<BITS, 128>(mp, grid, dev, stream);
    default: return fail(QMV_ERR_UNSUPPORTED, "group_size=%d on the tensor-core path", gs);
  }
}

int launch_mma(const void *x, const uint32_t *w, const void *scales,
               const void *biases, void *y, int M, int N, int K, int bits, int gs,
               DeviceInfo *dev, cudaStream_t stream, bool fixed_scratch) {
  qmvk::MmaParams mp;
  std::memset(&mp, 0, sizeof mp);
  mp.w = reinterpret_cast<const uint8_t *>(w);
  mp.s = static_cast<const uint16_t *>(scales);
  mp.b = static_cast<const uint16_t *>(biases);
  mp.x = static_cast<const uint16_t *>(x);
  mp.y = static_cast<uint16_t *>(y);
  mp.M = M;
  mp.N = N;
  mp.K = K;
  mp.G = K / gs;
  mp.row_bytes = static_cast<uint32_t>(static_cast<long long>(K) * bits / 8);
  mp.ntiles = (N + qmvk::kMmaRows - 1) / qmvk::kMmaRows;
  mp.nstage = K / (1024 / bits);
  mp.nsteps = static_cast<long long>(mp.ntiles) * mp.nstage;
  mp.k_magic = 0x64006400u;
  for (int i = 0; i < 3; ++i) {
    const uint32_t a = 0x8000u | (static_cast<uint32_t>(25 - (2 * i + 2)) << 10);
    mp.k_add[i] = a | (a << 16);
  }
  // one whole tile per CTA when the tiles fit the SMs; otherwise every SM
  // takes an equal share of the (tile, stage) steps (tiles cut between CTAs
  // are added up through the scratch slots)
  const int grid = mp.ntiles <= dev->sms ? mp.ntiles : dev->sms;
  int d = 0;
  cudaGetDevice(&d);
  MmaScratch *sc = nullptr;
  int rc;
  if ((rc = fixed_scratch ? static_scratch(d, dev->sms, mp.ntiles, &sc)
                         : mma_scratch(d,
                                       static_cast<size_t>(dev->sms) * 2 * qmvk::kMmaCols *
                                           qmvk::kMmaRows * sizeof(float),
                                       mp.ntiles, stream, &sc)))
    return rc;
  mp.part = sc->part;
  mp.cnt = sc->cnt;
  mp.err = dev->status;
  switch (bits) {
    case 2: return launch_mma_b<2>(mp, gs, grid, dev, stream);
    case 4: return launch_mma_b<4>(mp, gs, grid, dev, stream);
    case 8: return launch_mma_b<8>(mp, gs, grid, dev, stream);
    default: return fail(QMV_ERR_UNSUPPORTED, "bits=%d on the tensor-core path", bits);
  }
}

// ---------------------------------------------------------------------------
// Many activation rows (M > 16) on the tensor cores (qmv_qmm.cu): bf16
// operands, x straight from memory; the same code widths and shape rules as
// the few-row path.
// ---------------------------------------------------------------------------
constexpr long long kQmmMaxTiles = 1LL << 24;

bool qmm_path(int M, int N, int K, int bits, int gs) {
  if (!(bits == 2 || bits == 4 || bits == 8)) return false;
  if (!(gs == 32 || gs == 64 || gs == 128)) return false;
  return M >= kQmmMinRows && M >= kMmaMinRows && K % qmvq::qmm_stage_codes(bits) == 0 &&
         (K / gs) % 8 == 0 && qmvq::qmm_tiles(M, N) <= kQmmMaxTiles;
}

int launch_qmm(const void *x, const uint32_t *w, const void *scales, const void *biases,
               void *y, int M, int N, int K, int bits, int gs, DeviceInfo *dev,
               cudaStream_t stream, bool fixed_scratch) {
  qmvq::QmmArgs a;
  a.x = x;
  a.w = w;
  a.scales = scales;
  a.biases = biases;
  a.y = y;
  a.M = M;
  a.N = N;
  a.K = K;
  a.bits = bits;
  a.gs = gs;
  a.sms = dev->sms;
  a.smem_optin = dev->smem_optin;
  a.err = dev->status;
  a.part = nullptr;
  a.cnt = nullptr;
  a.stream = stream;
  if (!fixed_scratch) {
    // split tiles need the partial-sum slots and tile counters; without
    // scratch (qmv_noalloc) every CTA takes whole tiles
    int d = 0;
    cudaGetDevice(&d);
    MmaScratch *sc = nullptr;
    int rc;
    if ((rc = mma_scratch(d, qmvq::qmm_part_bytes(M, dev->sms),
                          static_cast<int>(qmvq::qmm_tiles(M, N)), stream, &sc)))
      return rc;
    a.part = sc->part;
    a.cnt = sc->cnt;
  }
  char msg[256];
  const int rc = qmvq::qmm_launch(a, msg, sizeof msg);
  if (rc) return fail(rc, "%s", msg);
  return ok();
}

int qmv_impl(const char *name, const void *x, const uint32_t *w, const void *scales,
             const void *biases, void *y, int M, int N, int K, int bits, int group_size,
             void *stream, bool fixed_scratch) {
  if (!x || !w || !scales || !biases || !y)
    return fail(QMV_ERR_NULL, "%s: a buffer pointer is NULL", name);
  int rc = check_common(N, K, bits, group_size);
  if (rc) return rc;
  if (M <= 0) return fail(QMV_ERR_SHAPE, "%s: M=%d must be positive", name, M);
  if (!aligned16(x) || !aligned16(w) || !aligned16(scales) ||
      !aligned16(biases) || !aligned16(y))
    return fail(QMV_ERR_ALIGN, "%s: buffers must be 16-byte aligned", name);
  DeviceInfo *dev;
  if ((rc = device_info(&dev))) return rc;
  if (mma_path(M, K, bits, group_size))
    return launch_mma(x, w, scales, biases, y, M, N, K, bits, group_size, dev,
                      static_cast<cudaStream_t>(stream), fixed_scratch);
  if (qmm_path(M, N, K, bits, group_size))
    return launch_qmm(x, w, scales, biases, y, M, N, K, bits, group_size, dev,
                      static_cast<cudaStream_t>(stream), fixed_scratch);
  if (decode_path(M, K, bits)) {
    DecodePlan dp;
    init_decode(dp, x, N, K, 1, dev);
    dp.p.w[0] = reinterpret_cast<const uint8_t *>(w);
    dp.p.s[0] = static_cast<const uint16_t *>(scales);
    dp.p.b[0] = static_cast<const uint16_t *>(biases);
    dp.p.y[0] = static_cast<uint16_t *>(y);
    if (make_decode_plan(dp, bits, group_size, false, dev))
      return launch_decode<false>(dp, bits, group_size, static_cast<cudaStream_t>(stream));
  }
  Plan pl;
  init_params(pl.p);
  qmvk::StreamParams &p = pl.p;
  p.mode = qmvk::MODE_QMV;
  p.w[0] = reinterpret_cast<const uint8_t *>(w);
  p.s[0] = static_cast<const uint16_t *>(scales);
  p.b[0] = static_cast<const uint16_t *>(biases);
  p.y[0] = static_cast<uint16_t *>(y);
  p.x = static_cast<const uint16_t *>(x);
  p.M = M;
  p.N = N;
  p.K = K;
  p.nmat = 1;
  p.total_rows = N;
  p.err = dev->status;
  if ((rc = make_plan(pl, bits, group_size, M, dev))) return rc;
  return launch(pl, bits, static_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------
// qvm (qmv_qvm.cuh)
// ---------------------------------------------------------------------------
template <int BITS>
int launch_qvm_t(const qmvk::QvmParams &p, cudaStream_t stream) {
  const int nblk = (p.N + qmvk::kQvmCols - 1) / qmvk::kQvmCols;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nblk, qmvk::kQvmCluster, p.M);
  cfg.blockDim = dim3(qmvk::kQvmWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t le = cudaLaunchKernelEx(&cfg, qmvk::qvm_kernel<BITS>, p);
  if (le != cudaSuccess) {
    cudaGetLastError();  // clear it
    return fail(QMV_ERR_CUDA, "qvm launch: %s", cudaGetErrorString(le));
  }
  return ok();
}

// The staged qvm: rows streamed by the tensor-copy engine.  Needs the code
// and scale rows to be multiples of 16 bytes (N * bits % 128 == 0 and
// (N / gs) % 8 == 0); other shapes take qvm_kernel.
// Dynamic shared memory of the staged qvm: the CTA's activations (fp32),
// 128 bytes of alignment slack, the stages.
// Rows of a column block are split between the CTAs of one cluster: 16 where
// the device allows clusters that large (twice the CTAs in flight), else 8.
constexpr int kQvtClusterBig = 16;

int qvm_tma_smem(int K, int bits, uint32_t *ring_off, uint32_t *stage_bytes) {
  const int xrows = (K + qmvk::kQvmCluster - 1) / qmvk::kQvmCluster + 1;
  *ring_off = static_cast<uint32_t>((4LL * xrows + 127) / 128 * 128);
  *stage_bytes = static_cast<uint32_t>(qmvk::kQvtRows * 32 * bits + 2 * qmvk::kQvtRows * 16);
  return static_cast<int>(*ring_off) + 128 + qmvk::kQvtStages * static_cast<int>(*stage_bytes);
}
// the staged kernel's static shared memory (partials, barriers), with room
constexpr int kQvtStaticSmem = 20 * 1024;

template <int BITS>
int launch_qvm_tma_t(const qmvk::QvmParams &q, DeviceInfo *dev, cudaStream_t stream) {
  constexpr int WB = 32 * BITS;
  qmvk::QvtParams p;
  std::memset(&p, 0, sizeof p);
  p.y = q.y;
  p.x = q.x;
  p.err = dev->status;
  p.M = q.M;
  p.K = q.K;
  p.N = q.N;
  p.gs_shift = q.gs_shift;
  p.x_off = 0;
  const int smem = qvm_tma_smem(q.K, BITS, &p.ring_off, &p.stage_bytes);
  CUtensorMap tw, ts, tb;
  int rc;
  if ((rc = encode_2d(&tw, q.w, CU_TENSOR_MAP_DATA_TYPE_UINT8, q.row_bytes, q.K, q.row_bytes, WB,
                      qmvk::kQvtRows, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B)))
    return rc;
  if ((rc = encode_2d(&ts, q.s, CU_TENSOR_MAP_DATA_TYPE_UINT16, q.G, q.K, 2ull * q.G, 8,
                      qmvk::kQvtRows, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B)))
    return rc;
  if ((rc = encode_2d(&tb, q.b, CU_TENSOR_MAP_DATA_TYPE_UINT16, q.G, q.K, 2ull * q.G, 8,
                      qmvk::kQvtRows, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B)))
    return rc;
  auto kern = qmvk::qvm_tma_kernel<BITS>;
  int d = 0;
  cudaGetDevice(&d);
  static int granted[kMaxDevices] = {};
  if (smem > 48 * 1024 && smem > granted[d]) {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
      return fail(QMV_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    granted[d] = smem;
  }
  const int nblk = (q.N + qmvk::kQvmCols - 1) / qmvk::kQvmCols;
  // the larger cluster where the device can hold one at this size (asked
  // once per device), else the portable size
  static int big_ok[kMaxDevices] = {};  // 0 unknown, 1 yes, 2 no
  if (!big_ok[d]) {
    big_ok[d] = 2;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
        cudaSuccess) {
      cudaLaunchConfig_t oc = {};
      oc.gridDim = dim3(nblk, kQvtClusterBig, 1);
      oc.blockDim = dim3((qmvk::kQvtWarps + 1) * 32);
      oc.dynamicSmemBytes = static_cast<size_t>(smem);
      cudaLaunchAttribute ca[1];
      ca[0].id = cudaLaunchAttributeClusterDimension;
      ca[0].val.clusterDim.x = 1;
      ca[0].val.clusterDim.y = kQvtClusterBig;
      ca[0].val.clusterDim.z = 1;
      oc.attrs = ca;
      oc.numAttrs = 1;
      int nc = 0;
      if (cudaOccupancyMaxActiveClusters(&nc, kern, &oc) == cudaSuccess && nc >= 1) big_ok[d] = 1;
    }
    cudaGetLastError();  // a refused size leaves no error behind
  }
  const int ncl = big_ok[d] == 1 ? kQvtClusterBig : qmvk::kQvmCluster;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nblk, ncl, q.M);
  cfg.blockDim = dim3((qmvk::kQvtWarps + 1) * 32);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 1;
  attr[1].val.clusterDim.y = ncl;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t le = cudaLaunchKernelEx(&cfg, kern, tw, ts, tb, p);
  if (le != cudaSuccess) {
    cudaGetLastError();  // clear it
    return fail(QMV_ERR_CUDA, "qvm launch: %s", cudaGetErrorString(le));
  }
  return ok();
}

// ---------------------------------------------------------------------------
// Trellis mode (qmv_trellis.cuh)
// ---------------------------------------------------------------------------
template <int BITS>
int launch_trellis_t(const qmvk::TrellisParams &p, int sms, cudaStream_t stream) {
  auto kern = qmvk::qmv_trellis_kernel<BITS>;
  const int smem = 4 * p.K;
  int dev = 0;
  cudaGetDevice(&dev);
  static int granted[kMaxDevices] = {};
  if (smem > 48 * 1024 && smem > granted[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess)
      return fail(QMV_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    granted[dev] = smem;
  }
  const int rows_per_cta = qmvk::kTrellisWarps * qmvk::trellis_rows_per_warp<BITS>();
  long long grid = (p.N + rows_per_cta - 1) / rows_per_cta;
  if (grid > 16LL * sms) grid = 16LL * sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), p.M);
  cfg.blockDim = dim3(qmvk::kTrellisWarps * 32);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t le = cudaLaunchKernelEx(&cfg, kern, p);
  if (le != cudaSuccess) {
    cudaGetLastError();  // clear it
    return fail(QMV_ERR_CUDA, "qmv_trellis launch: %s", cudaGetErrorString(le));
  }
  return ok();
}

}  // namespace

extern "C" {

int qmv_abi_version(void) { return 1; }

int qmv_device_status(int *out, int reset, void *stream) {
  if (!out) return fail(QMV_ERR_NULL, "qmv_device_status: out is NULL");
  DeviceInfo *dev;
  int rc;
  if ((rc = device_info(&dev))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(out, dev->status, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && reset) e = cudaMemsetAsync(dev->status, 0, sizeof(int), st);
  if (e != cudaSuccess) return fail(QMV_ERR_CUDA, "qmv_device_status: %s", cudaGetErrorString(e));
  return ok();
}

const char *qmv_last_error(void) { return g_last_error.c_str(); }

int qmv(const void *x, const uint32_t *w, const void *scales,
        const void *biases, void *y, int M, int N, int K, int bits,
        int group_size, void *stream) {
  return qmv_impl("qmv", x, w, scales, biases, y, M, N, K, bits, group_size, stream, false);
}

int qmv_noalloc(const void *x, const uint32_t *w, const void *scales, const void *biases,
                void *y, int M, int N, int K, int bits, int group_size, void *stream) {
  return qmv_impl("qmv_noalloc", x, w, scales, biases, y, M, N, K, bits, group_size, stream,
                  true);
}

int qvm(const void *x, const uint32_t *w, const void *scales, const void *biases, void *y,
        int M, int K, int N, int bits, int group_size, void *stream) {
  if (!x || !w || !scales || !biases || !y)
    return fail(QMV_ERR_NULL, "qvm: a buffer pointer is NULL");
  // W has K rows of N codes; the groups run along N (the output axis)
  if (!bits_supported(bits))
    return fail(QMV_ERR_UNSUPPORTED, "qvm: bits=%d not in {2,3,4,5,6,8}", bits);
  if (!gs_supported(group_size))
    return fail(QMV_ERR_UNSUPPORTED, "qvm: group_size=%d not in {32,64,128}", group_size);
  if (K <= 0 || N <= 0) return fail(QMV_ERR_SHAPE, "qvm: K=%d and N=%d must be positive", K, N);
  if (N % group_size != 0)
    return fail(QMV_ERR_SHAPE, "qvm: N=%d is not a multiple of group_size=%d", N, group_size);
  int rc;
  if (M <= 0) return fail(QMV_ERR_SHAPE, "qvm: M=%d must be positive", M);
  if (M > 65535) return fail(QMV_ERR_UNSUPPORTED, "qvm: M=%d above 65535", M);
  const void *ptrs[] = {x, w, scales, biases, y};
  for (const void *q : ptrs)
    if (!aligned16(q)) return fail(QMV_ERR_ALIGN, "qvm: buffers must be 16-byte aligned");
  DeviceInfo *dev;
  if ((rc = device_info(&dev))) return rc;
  qmvk::QvmParams p;
  std::memset(&p, 0, sizeof p);
  p.w = reinterpret_cast<const uint8_t *>(w);
  p.s = static_cast<const uint16_t *>(scales);
  p.b = static_cast<const uint16_t *>(biases);
  p.x = static_cast<const uint16_t *>(x);
  p.y = static_cast<uint16_t *>(y);
  p.M = M;
  p.K = K;
  p.N = N;
  p.G = N / group_size;
  p.gs_shift = group_size == 32 ? 5 : group_size == 64 ? 6 : 7;
  p.row_bytes = static_cast<uint32_t>(static_cast<long long>(N) * bits / 8);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t ro, sbytes;
  if ((static_cast<long long>(N) * bits) % 128 == 0 && p.G % 8 == 0 &&
      qvm_tma_smem(K, bits, &ro, &sbytes) <= dev->smem_optin - kQvtStaticSmem) {
    switch (bits) {
      case 2: return launch_qvm_tma_t<2>(p, dev, st);
      case 3: return launch_qvm_tma_t<3>(p, dev, st);
      case 4: return launch_qvm_tma_t<4>(p, dev, st);
      case 5: return launch_qvm_tma_t<5>(p, dev, st);
      case 6: return launch_qvm_tma_t<6>(p, dev, st);
      case 8: return launch_qvm_tma_t<8>(p, dev, st);
      default: break;
    }
  }
  switch (bits) {
    case 2: return launch_qvm_t<2>(p, st);
    case 3: return launch_qvm_t<3>(p, st);
    case 4: return launch_qvm_t<4>(p, st);
    case 5: return launch_qvm_t<5>(p, st);
    case 6: return launch_qvm_t<6>(p, st);
    case 8: return launch_qvm_t<8>(p, st);
    default: return fail(QMV_ERR_UNSUPPORTED, "qvm: bits=%d", bits);
  }
}

int qmv_trellis(const void *x, const uint32_t *w, const void *scales, void *y, int M, int N,
                int K, int bits, void *stream) {
  if (!x || !w || !scales || !y)
    return fail(QMV_ERR_NULL, "qmv_trellis: a buffer pointer is NULL");
  if (bits != 2 && bits != 4)
    return fail(QMV_ERR_UNSUPPORTED, "qmv_trellis: bits=%d not in {2,4}", bits);
  if (M <= 0 || N <= 0 || K <= 0)
    return fail(QMV_ERR_SHAPE, "qmv_trellis: M=%d, N=%d, K=%d must be positive", M, N, K);
  if ((static_cast<long long>(K) * bits) % 128 != 0)
    return fail(QMV_ERR_SHAPE, "qmv_trellis: K*bits=%lld is not a multiple of 128",
                static_cast<long long>(K) * bits);
  if (K > 49152) return fail(QMV_ERR_UNSUPPORTED, "qmv_trellis: K=%d above 49152", K);
  if (M > 65535) return fail(QMV_ERR_UNSUPPORTED, "qmv_trellis: M=%d above 65535", M);
  const void *ptrs[] = {x, w, y};
  for (const void *q : ptrs)
    if (!aligned16(q))
      return fail(QMV_ERR_ALIGN, "qmv_trellis: buffers must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(scales) & 1u)
    return fail(QMV_ERR_ALIGN, "qmv_trellis: scales must be 2-byte aligned");
  DeviceInfo *dev;
  int rc;
  if ((rc = device_info(&dev))) return rc;
  qmvk::TrellisParams p;
  std::memset(&p, 0, sizeof p);
  p.w = reinterpret_cast<const uint16_t *>(w);
  p.x = static_cast<const uint16_t *>(x);
  p.scales = static_cast<const uint16_t *>(scales);
  p.y = static_cast<uint16_t *>(y);
  p.M = M;
  p.N = N;
  p.K = K;
  p.W = static_cast<int>(static_cast<long long>(K) * bits / 16);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return bits == 2 ? launch_trellis_t<2>(p, dev->sms, st) : launch_trellis_t<4>(p, dev->sms, st);
}

int qmv_gate_up(const void *x, const uint32_t *w_gate, const void *s_gate,
                const void *b_gate, const uint32_t *w_up, const void *s_up,
                const void *b_up, void *y_gate, void *y_up, int M, int N,
                int K, int bits, int group_size, void *stream) {
  if (!x || !w_gate || !s_gate || !b_gate || !w_up || !s_up || !b_up ||
      !y_gate || !y_up)
    return fail(QMV_ERR_NULL, "qmv_gate_up: a buffer pointer is NULL");
  int rc = check_common(N, K, bits, group_size);
  if (rc) return rc;
  if (M <= 0) return fail(QMV_ERR_SHAPE, "qmv_gate_up: M=%d must be positive", M);
  if (N > (1 << 30))
    return fail(QMV_ERR_UNSUPPORTED, "qmv_gate_up: N=%d above 2^30", N);
  const void *ptrs[] = {x, w_gate, s_gate, b_gate, w_up, s_up, b_up, y_gate, y_up};
  for (const void *q : ptrs)
    if (!aligned16(q))
      return fail(QMV_ERR_ALIGN, "qmv_gate_up: buffers must be 16-byte aligned");
  DeviceInfo *dev;
  if ((rc = device_info(&dev))) return rc;
  if (decode_path(M, K, bits)) {
    DecodePlan dp;
    init_decode(dp, x, N, K, 2, dev);
    dp.p.w[0] = reinterpret_cast<const uint8_t *>(w_gate);
    dp.p.s[0] = static_cast<const uint16_t *>(s_gate);
    dp.p.b[0] = static_cast<const uint16_t *>(b_gate);
    dp.p.y[0] = static_cast<uint16_t *>(y_gate);
    dp.p.w[1] = reinterpret_cast<const uint8_t *>(w_up);
    dp.p.s[1] = static_cast<const uint16_t *>(s_up);
    dp.p.b[1] = static_cast<const uint16_t *>(b_up);
    dp.p.y[1] = static_cast<uint16_t *>(y_up);
    if (make_decode_plan(dp, bits, group_size, false, dev))
      return launch_decode<false>(dp, bits, group_size, static_cast<cudaStream_t>(stream));
  }
  Plan pl;
  init_params(pl.p);
  qmvk::StreamParams &p = pl.p;
  p.mode = qmvk::MODE_GATE_UP;
  p.w[0] = reinterpret_cast<const uint8_t *>(w_gate);
  p.s[0] = static_cast<const uint16_t *>(s_gate);
  p.b[0] = static_cast<const uint16_t *>(b_gate);
  p.y[0] = static_cast<uint16_t *>(y_gate);
  p.w[1] = reinterpret_cast<const uint8_t *>(w_up);
  p.s[1] = static_cast<const uint16_t *>(s_up);
  p.b[1] = static_cast<const uint16_t *>(b_up);
  p.y[1] = static_cast<uint16_t *>(y_up);
  p.x = static_cast<const uint16_t *>(x);
  p.M = M;
  p.N = N;
  p.K = K;
  p.nmat = 2;
  p.total_rows = N;
  p.err = dev->status;
  if ((rc = make_plan(pl, bits, group_size, M, dev))) return rc;
  return launch(pl, bits, static_cast<cudaStream_t>(stream));
}

int qmv_silu_gate_resid(const void *gate, const void *up, const void *x_resid,
                        const uint32_t *w, const void *scales,
                        const void *biases, void *y, int M, int N, int K,
                        int bits, int group_size, void *stream) {
  if (!gate || !up || !w || !scales || !biases || !y)
    return fail(QMV_ERR_NULL, "qmv_silu_gate_resid: a buffer pointer is NULL");
  int rc = check_common(N, K, bits, group_size);
  if (rc) return rc;
  if (M <= 0)
    return fail(QMV_ERR_SHAPE, "qmv_silu_gate_resid: M=%d must be positive", M);
  const void *ptrs[] = {gate, up, w, scales, biases, y};
  for (const void *q : ptrs)
    if (!aligned16(q))
      return fail(QMV_ERR_ALIGN,
                  "qmv_silu_gate_resid: buffers must be 16-byte aligned");
  if (x_resid && (reinterpret_cast<uintptr_t>(x_resid) & 1u))
    return fail(QMV_ERR_ALIGN, "qmv_silu_gate_resid: x_resid must be 2-byte aligned");
  DeviceInfo *dev;
  if ((rc = device_info(&dev))) return rc;
  if (decode_path(M, K, bits)) {
    DecodePlan dp;
    init_decode(dp, gate, N, K, 1, dev);
    dp.p.up = static_cast<const uint16_t *>(up);
    dp.p.resid = static_cast<const uint16_t *>(x_resid);
    dp.p.w[0] = reinterpret_cast<const uint8_t *>(w);
    dp.p.s[0] = static_cast<const uint16_t *>(scales);
    dp.p.b[0] = static_cast<const uint16_t *>(biases);
    dp.p.y[0] = static_cast<uint16_t *>(y);
    if (make_decode_plan(dp, bits, group_size, true, dev))
      return launch_decode<true>(dp, bits, group_size, static_cast<cudaStream_t>(stream));
  }
  Plan pl;
  init_params(pl.p);
  qmvk::StreamParams &p = pl.p;
  p.mode = qmvk::MODE_SILU;
  p.w[0] = reinterpret_cast<const uint8_t *>(w);
  p.s[0] = static_cast<const uint16_t *>(scales);
  p.b[0] = static_cast<const uint16_t *>(biases);
  p.y[0] = static_cast<uint16_t *>(y);
  p.x = static_cast<const uint16_t *>(gate);
  p.up = static_cast<const uint16_t *>(up);
  p.resid = static_cast<const uint16_t *>(x_resid);
  p.M = M;
  p.N = N;
  p.K = K;
  p.nmat = 1;
  p.total_rows = N;
  p.err = dev->status;
  if ((rc = make_plan(pl, bits, group_size, M, dev))) return rc;
  return launch(pl, bits, static_cast<cudaStream_t>(stream));
}

int gather_qmv(const void *x, const uint32_t *w, const void *scales,
               const void *biases, const uint32_t *lhs_indices,
               const uint32_t *rhs_indices, void *y, int num_pairs,
               int num_x_rows, int num_experts, int N, int K, int bits,
               int group_size, int sorted_indices, int *d_status,
               void *stream) {
  (void)sorted_indices;  // grouping by expert happens on the device either way
  if (!x || !w || !scales || !biases || !rhs_indices || !y)
    return fail(QMV_ERR_NULL, "gather_qmv: a buffer pointer is NULL");
  int rc = check_common(N, K, bits, group_size);
  if (rc) return rc;
  if (num_pairs < 0 || num_x_rows <= 0 || num_experts <= 0)
    return fail(QMV_ERR_SHAPE,
                "gather_qmv: num_pairs=%d num_x_rows=%d num_experts=%d",
                num_pairs, num_x_rows, num_experts);
  if (!lhs_indices && num_x_rows < num_pairs)
    return fail(QMV_ERR_SHAPE,
                "gather_qmv: without lhs_indices num_x_rows must be >= num_pairs");
  if (static_cast<long long>(num_experts) * N > 0x7fffffffLL)
    return fail(QMV_ERR_UNSUPPORTED, "gather_qmv: num_experts * N above 2^31");
  if (3LL * num_experts + num_pairs > 24576)
    return fail(QMV_ERR_UNSUPPORTED,
                "gather_qmv: num_pairs + 3*num_experts above 24576");
  if (num_pairs == 0) return ok();
  const void *ptrs[] = {x, w, scales, biases, y};
  for (const void *q : ptrs)
    if (!aligned16(q))
      return fail(QMV_ERR_ALIGN, "gather_qmv: buffers must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(rhs_indices) & 3u) ||
      (reinterpret_cast<uintptr_t>(lhs_indices) & 3u) ||
      (reinterpret_cast<uintptr_t>(d_status) & 3u))
    return fail(QMV_ERR_ALIGN, "gather_qmv: index arrays must be 4-byte aligned");
  DeviceInfo *dev;
  if ((rc = device_info(&dev))) return rc;
  Plan pl;
  init_params(pl.p);
  qmvk::StreamParams &p = pl.p;
  p.mode = qmvk::MODE_GATHER;
  p.w[0] = reinterpret_cast<const uint8_t *>(w);
  p.s[0] = static_cast<const uint16_t *>(scales);
  p.b[0] = static_cast<const uint16_t *>(biases);
  p.y[0] = static_cast<uint16_t *>(y);
  p.x = static_cast<const uint16_t *>(x);
  p.lhs = lhs_indices;
  p.rhs = rhs_indices;
  p.status = d_status;
  p.M = 1;
  p.N = N;
  p.K = K;
  p.nmat = 1;
  p.num_pairs = num_pairs;
  p.num_x_rows = num_x_rows;
  p.num_experts = num_experts;
  p.total_rows = static_cast<long long>(num_experts) * N;
  // a bounded wait that gives up is reported in the caller's status word
  // when there is one
  p.err = d_status ? d_status : dev->status;
  const int mr = num_pairs >= num_experts ? 2 : 1;
  if ((rc = make_plan(pl, bits, group_size, mr, dev))) return rc;
  return launch(pl, bits, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
