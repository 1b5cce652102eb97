// C ABI of the CODA GEMM + epilogue hot path (declarations and contracts in
// include/coda.h).  Host side: argument validation (before any CUDA call),
// tensor-map encoding, and launches on the caller's stream.  The library keeps
// no device allocations of its own.
#include <algorithm>
#include <mutex>

#include <cmath>

#include "coda.h"
#include "coda_device.cuh"
#include "coda_block.cuh"
#include "coda_gemm.cuh"
#include "coda_grouped.cuh"
#include "coda_rowops.cuh"

namespace {

using namespace coda;

constexpr int64_t kPartialTile = 128;  // columns per partial sum: one half of a 256-column tile
constexpr int kVersion = 3;  // 2: partial sums per 128-column slot; 3: the MXFP8 calls

int64_t g_wait_ns = 1000000000LL;

// --------------------------------------------------------------- validation

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool dim_ok(int64_t v) { return v > 0 && (v % 8) == 0 && v <= (int64_t(1) << 31) - 1; }

#define CODA_CHECK(cond, code) \
  do {                         \
    if (!(cond)) return code;  \
  } while (0)

// ------------------------------------------------------------------ devices

struct DevInfo {
  bool init = false;
  bool ok = false;
  int sms = 0;
  uint32_t attr_set = 0;  // bit per kernel kind: dynamic smem attribute applied
};

std::mutex g_mu;
DevInfo g_dev[64];

coda_status_t current_device(int* dev_out, DevInfo** info) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return CODA_ERR_DEVICE;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  DevInfo& d = g_dev[dev];
  if (!d.init) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return CODA_ERR_DEVICE;
    }
    d.init = true;
    d.ok = (major == 10 && minor == 0);
    d.sms = sms;
  }
  if (!d.ok) return CODA_ERR_DEVICE;
  *dev_out = dev;
  *info = &d;
  return CODA_OK;
}

// -------------------------------------------------------------- tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// 2-D row-major tensor [rows, cols] with row stride `stride` elements; box
// box_cols x box_rows; 128-byte swizzle; out-of-range elements read as zero.
bool tmap2d(CUtensorMap* m, const void* base, bool f32, uint64_t cols, uint64_t rows, uint64_t stride,
            uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const uint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {stride * es};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// e4m3 operands and outputs: 1-byte elements, 128-byte inner boxes (one swizzle row).
bool tmap2d_u8(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t stride,
               uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {stride};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// e4m3 output rows of 64 bytes without swizzle (staged as plain rows).
bool tmap2d_u8_plain(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t stride,
                     uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {stride};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Scale bytes of a block-scaled operand seen as rows of 128 32-bit words
// (512 bytes), `box_rows` rows per copy.
bool tmap_sf(CUtensorMap* m, const void* base, uint64_t atoms, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {128, atoms};
  cuuint64_t strides[1] = {512};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Operand maps of the mainloop.  A: [M, K] K-major (box 64 x 128) or stored
// transposed as [K, M] (MN-major, box 64 x 64).  B: [K, N] MN-major (box 64 x 64)
// or stored transposed as [N, K] (K-major, box 64 x BN).
bool map_a(CUtensorMap* m, const void* p, bool mn, uint64_t M, uint64_t K) {
  return mn ? tmap2d(m, p, false, M, K, M, 64, kBK) : tmap2d(m, p, false, K, M, K, kBK, kBM);
}
bool map_b(CUtensorMap* m, const void* p, bool mn, uint64_t N, uint64_t K, uint64_t stride, uint32_t bn) {
  return mn ? tmap2d(m, p, false, N, K, stride, 64, kBK) : tmap2d(m, p, false, K, N, stride, kBK, bn);
}
// Epilogue tile maps: 32 rows per warp, 128-byte rows.
bool map_out_bf16(CUtensorMap* m, const void* p, uint64_t rows, uint64_t cols, uint64_t stride) {
  return tmap2d(m, p, false, cols, rows, stride, 64, 32);
}
bool map_out_f32(CUtensorMap* m, const void* p, uint64_t rows, uint64_t cols) {
  return tmap2d(m, p, true, cols, rows, cols, 32, 32);
}
bool map_out_f32_ld(CUtensorMap* m, const void* p, uint64_t rows, uint64_t cols, uint64_t stride) {
  return tmap2d(m, p, true, cols, rows, stride, 32, 32);
}

// ------------------------------------------------------------------ launch

enum KernelKind : uint32_t {
  kKindResPartial = 0,
  kKindRowScale,
  kKindRowScaleKK,
  kKindSwiGLU,
  kKindSwiGLUAct,     // the SwiGLU GEMM without the gate/up save
  kKindCE,
  kKindBwdP,
  kKindF32MN,
  kKindSwiGLUBwd,
  kKindCEGrad,
  kKindF32KK,
  kKindRope,
  kKindBlock,
  kKindResPartialF8,
  kKindRowScaleF8,
  kKindResPartialMX,
  kKindRowScaleMX,
  kKindGroupedCE,      // CE backward: dW (long) + dH
  kKindGroupedWX,      // first-GEMM backward: dW1 (long) + dx
  kKindCount
};

// Vocabulary columns per chunk of the cross-entropy backward: the chunk's
// bf16 gradient (M x 8192) is written once and read by two GEMMs right after.
// (Interleaved on one B200 at 8192 x 2048 x 128256: 2048 columns 12.4 ms,
// 4096 10.9, 8192 10.5, 16384 10.8: wider chunks halve the launches and the
// fp32 dH accumulations; 16384-column gradients no longer fit in L2.)
constexpr int64_t kCEBwdChunk = 8192;

// Pipeline depth of the pair kernels: as many 32 KB stages (this CTA's halves
// of A and B, plus 1.5 KB of scales for block-scaled operands) as fit next to
// the epilogue's shared memory, at most 8.
template <class Epi>
constexpr int pair_stages() {
  constexpr int budget = 232448 - 1024 - 256 - GemmSmem<256, 1, true, Epi>::kEpiBytes -
                         GemmSmem<256, 1, true, Epi>::kXchgBytes;
  constexpr int st = budget / (2 * kBM * kBK * 2 + GemmSmem<256, 1, true, Epi>::kSFStage);
  return st > 8 ? 8 : st;
}

// Raster order.  The tiles that run at the same time should share the operand
// that stays resident in L2, so that the other operand streams from DRAM once:
//   A (M x K) no larger than B (K x N): every M tile of a column block runs
//     before the next column block (group = all rows): A stays resident and
//     each column block of B is read once.  An A of more than 40 MiB (bf16)
//     does not stay in L2 (126 MB) beside B's column blocks and the output
//     streaming through it; then the M tiles go in groups whose rows of A
//     take 32 MiB, each group sweeping all column blocks (B is read once per
//     group).  At hidden 4096 (A 64 MiB) the second GEMM took 1210 against
//     1292 us that way, at hidden 8192 (128 MiB) the first 731 against 777
//     and the second 6925 against 7053 us;
//   otherwise row-major order (group = 1): B stays resident and each row
//     block of A is read once.
constexpr int kAllRows = 1 << 30;

inline int raster_group(int64_t M, int64_t N, int64_t K) {
  if (M * K > N * K) return 1;
  if (M * K * 2 <= (int64_t(40) << 20)) return kAllRows;
  const int64_t g = (int64_t(32) << 20) / (2 * kBM * K * 2);  // rows of A per pair tile: 2 kBM
  return g < 1 ? 1 : static_cast<int>(g);
}

struct KernelCache {
  bool attr = false;
  int max_clusters = 0;  // resident clusters of two CTAs (pair kernels)
};
KernelCache g_kcache[64][32];
static_assert(kKindCount <= 32, "kernel kinds fit the cache");

// An output that K-half units add into (TileSched::kmode): the host zeroes
// the part of it that the split tiles cover before the launch.  Element
// (i, j) of the layout is at base + i * pitch + j * elem; a GEMM tile (mb, nb)
// covers layout rows [mb * tile_rows, ...) and columns [nb * tile_cols, ...),
// or with `transposed` rows [nb * tile_rows, ...) and columns [mb * tile_cols, ...)
// (the per-slot row sums, [slot, row]).
struct ZeroPlan {
  void* base;
  size_t pitch, elem;
  int64_t rows, cols;
  int tile_rows, tile_cols;
  bool transposed;
};

// A K-split needs this many k-blocks (K >= 4096 bf16): then a half takes half
// of a tile's mainloop, where a 128-column half tile still takes 93-96 % of it.
constexpr int kKSplitMinKb = 64;

template <int BN, int STAGES, bool A_MN, bool B_MN, bool PAIR, class Epi>
coda_status_t run_gemm(int dev, DevInfo* info, GemmParams<Epi>& p, int M, int N, int K, int n_nt, int group_m,
                       KernelKind kind, cudaStream_t stream, const ZeroPlan* zp = nullptr, int nzp = 0) {
  auto kern = coda_gemm_kernel<BN, STAGES, A_MN, B_MN, PAIR, Epi>;
  constexpr int smem = GemmSmem<BN, STAGES, PAIR, Epi>::kBytes;
  constexpr int kTileM = PAIR ? 2 * kBM : kBM;
  constexpr int kThr = 64 + 32 * epi_warps<Epi>::value;  // producer + MMA warps, epilogue warps
  KernelCache& kc = g_kcache[dev][kind];
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!kc.attr) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return CODA_ERR_LAUNCH;
      if (PAIR) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2 * (info->sms / 2), 1, 1);
        cfg.blockDim = dim3(kThr, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
          cudaGetLastError();
          n = info->sms / 2;
        }
        kc.max_clusters = n;
      }
      kc.attr = true;
    }
  }
  p.M = M;
  p.N = N;
  p.K = K;
  p.sched.n_mt = (M + kTileM - 1) / kTileM;
  p.sched.n_nt = n_nt;
  p.sched.group_m = group_m < 1 ? 1 : (group_m > p.sched.n_mt ? p.sched.n_mt : group_m);
  p.sched.ntiles = p.sched.n_mt * n_nt;
  p.wait_ns = static_cast<uint64_t>(g_wait_ns);
  if (!PAIR) {
    const int grid = p.sched.ntiles < info->sms ? p.sched.ntiles : info->sms;
    kern<<<grid, kThr, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? CODA_OK : CODA_ERR_LAUNCH;
  }
  // A last partial wave of whole tiles that fills at most half of the CTA
  // pairs runs as a wave of half units on twice as many pairs: e.g. 256
  // tiles on 74 pairs end in 34 tiles, 3.46 waves taking four tile-times.
  // (A grid of fewer tiles than pairs is one such wave: all of its tiles are
  // halved.)  Halves of the k-blocks, for epilogues whose fp32 outputs are
  // linear in the accumulator and long K: each runs half of the tile's
  // mainloop at full width and adds into the output zeroed here; otherwise
  // 128-column halves, whose MMAs still take 93-96 % of a whole tile's time
  // (they are bound by operand delivery, not by the tensor pipe).
  p.sched.nsplit = 0;
  p.sched.kmode = 0;
  {
    const int last = p.sched.ntiles % kc.max_clusters;
    constexpr int kKbElems = epi_fp8<Epi>::value ? 2 * kBK : kBK;
    const int nkb = (K + kKbElems - 1) / kKbElems;
    if (last > 0 && 2 * last <= kc.max_clusters) {
      if (epi_ksplit<Epi>::value && nzp > 0 && nkb >= kKSplitMinKb) {
        int mb0 = p.sched.n_mt, mb1 = -1, nb0 = n_nt, nb1 = -1;
        for (int t = p.sched.ntiles - last; t < p.sched.ntiles; ++t) {
          int mb, nb;
          p.sched.map(t, mb, nb);
          mb0 = mb < mb0 ? mb : mb0;
          mb1 = mb > mb1 ? mb : mb1;
          nb0 = nb < nb0 ? nb : nb0;
          nb1 = nb > nb1 ? nb : nb1;
        }
        for (int i = 0; i < nzp; ++i) {
          const ZeroPlan& z = zp[i];
          const int a0 = z.transposed ? nb0 : mb0, a1 = z.transposed ? nb1 : mb1;
          const int b0 = z.transposed ? mb0 : nb0, b1 = z.transposed ? mb1 : nb1;
          const int64_t r0 = static_cast<int64_t>(a0) * z.tile_rows;
          const int64_t r1 = std::min<int64_t>(static_cast<int64_t>(a1 + 1) * z.tile_rows, z.rows);
          const int64_t c0 = static_cast<int64_t>(b0) * z.tile_cols;
          const int64_t c1 = std::min<int64_t>(static_cast<int64_t>(b1 + 1) * z.tile_cols, z.cols);
          if (r1 <= r0 || c1 <= c0) continue;
          if (cudaMemset2DAsync(static_cast<uint8_t*>(z.base) + r0 * z.pitch + c0 * z.elem, z.pitch, 0,
                                static_cast<size_t>(c1 - c0) * z.elem, static_cast<size_t>(r1 - r0),
                                stream) != cudaSuccess)
            return CODA_ERR_LAUNCH;
        }
        p.sched.kmode = 1;
        p.sched.nsplit = last;
      } else if (epi_split<Epi>::value && (B_MN || p.has_bh)) {
        p.sched.nsplit = last;
      }
    }
  }
  const int units = p.sched.ntiles + p.sched.nsplit;
  const int clusters = units < kc.max_clusters ? units : kc.max_clusters;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(kThr, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // Programmatic dependent launch: this grid may start (prologue only) while
  // the previous kernel on the stream finishes, and waits for it in
  // griddepcontrol.wait; it lets the next one start likewise.
  cudaLaunchAttribute attr2[2];
  attr2[0] = attr[0];
  attr2[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr2[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr2;
  cfg.numAttrs = 2;
  p.pdl_wait = 1;
  p.pdl_trigger = 1;
  if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return CODA_ERR_LAUNCH;
  return cudaGetLastError() == cudaSuccess ? CODA_OK : CODA_ERR_LAUNCH;
}

// ---------------------------------------------------- grouped pair launch

template <class E0, class E1>
constexpr int grouped_stages() {
  constexpr int budget = 232448 - 1024 - 256 - GroupedSmem<E0, E1>::kEpiBytes;
  constexpr int st = budget / (2 * kBM * kBK * 2);
  return st > 8 ? 8 : st;
}

// The smallest makespan (k-blocks) at which the pairs' capacities, computed
// as the kernel computes them, take every tile of problem 1.
int grouped_target(int np, int n0, int n1, int u0, int u1) {
  const int lo = n0 / np;
  const int a = n0 - lo * np;
  const long total = static_cast<long>(n0) * u0 + static_cast<long>(n1) * u1;
  long t = (total + np - 1) / np;
  const long tmin = static_cast<long>(a > 0 ? lo + 1 : lo) * u0;
  if (t < tmin) t = tmin;
  for (;; ++t) {
    const long cap = static_cast<long>(a) * grouped_cap(static_cast<int>(t), lo + 1, u0, u1) +
                     static_cast<long>(np - a) * grouped_cap(static_cast<int>(t), lo, u0, u1);
    if (cap >= n1) return static_cast<int>(t);
  }
}

struct GroupedProblem {
  int M, N, K, group_m;
  bool a_mn, b_mn;
};

// Problem 0 must be the one with more k-blocks per tile.
template <class E0, class E1>
coda_status_t run_grouped(int dev, DevInfo* info, GroupedParams<E0, E1>& p, const GroupedProblem (&pb)[2],
                          KernelKind kind, cudaStream_t stream) {
  constexpr int STAGES = grouped_stages<E0, E1>();
  constexpr int smem = GroupedSmem<E0, E1>::template bytes<STAGES>();
  static_assert(smem <= 232448, "grouped kernel shared memory");
  auto kern = coda_gemm_grouped_kernel<256, STAGES, E0, E1>;
  KernelCache& kc = g_kcache[dev][kind];
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!kc.attr) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return CODA_ERR_LAUNCH;
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * (info->sms / 2), 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = info->sms / 2;
      }
      kc.max_clusters = n;
      kc.attr = true;
    }
  }
  for (int q = 0; q < 2; ++q) {
    p.M[q] = pb[q].M;
    p.N[q] = pb[q].N;
    p.K[q] = pb[q].K;
    p.n_mt[q] = (pb[q].M + 255) / 256;
    p.n_nt[q] = (pb[q].N + 255) / 256;
    p.group_m[q] = pb[q].group_m < 1 ? 1 : (pb[q].group_m > p.n_mt[q] ? p.n_mt[q] : pb[q].group_m);
    p.ntiles[q] = p.n_mt[q] * p.n_nt[q];
    p.a_mn[q] = pb[q].a_mn ? 1 : 0;
    p.b_mn[q] = pb[q].b_mn ? 1 : 0;
  }
  const int np = kc.max_clusters;
  p.target = grouped_target(np, p.ntiles[0], p.ntiles[1], (p.K[0] + kBK - 1) / kBK, (p.K[1] + kBK - 1) / kBK);
  p.wait_ns = static_cast<uint64_t>(g_wait_ns);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * np, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr2[2];  // programmatic dependent launch, as in run_gemm
  attr2[0] = attr[0];
  attr2[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr2[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr2;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return CODA_ERR_LAUNCH;
  return cudaGetLastError() == cudaSuccess ? CODA_OK : CODA_ERR_LAUNCH;
}

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

size_t ce_ws_bytes(int64_t M, int64_t V) {
  const int64_t n_nt = (V + 255) / 256;
  return 2 * align256(static_cast<size_t>(n_nt) * M * 4) + align256(static_cast<size_t>(M) * 4);
}

// The SwiGLU GEMM with (EpiSwiGLU) or without (EpiSwiGLUAct) the gate/up save.
template <class Epi>
coda_status_t run_swiglu(int dev, DevInfo* info, const uint16_t* A, const uint16_t* W_gu, const float* r,
                         uint16_t* act_out, uint16_t* gateup_save, int64_t M, int64_t F, int64_t K,
                         KernelKind kind, cudaStream_t stream) {
  GemmParams<Epi> p{};
  bool ok = map_a(&p.tmA, A, false, M, K) && map_b(&p.tmB, W_gu, true, F, K, 2 * F, 128) &&
            map_b(&p.tmB2, W_gu + F, true, F, K, 2 * F, 128) && map_out_bf16(&p.ep.tmAct, act_out, M, F, F);
  if (gateup_save)
    ok = ok && map_out_bf16(&p.ep.tmSaveG, gateup_save, M, F, 2 * F) &&
         map_out_bf16(&p.ep.tmSaveU, gateup_save + F, M, F, 2 * F);
  if (!ok) return CODA_ERR_INTERNAL;
  p.ep.r = r;
  const int n_nt = static_cast<int>((F + 127) / 128);
  return run_gemm<256, pair_stages<Epi>(), false, true, true, Epi>(dev, info, p, static_cast<int>(M), static_cast<int>(F),
                                                                    static_cast<int>(K), n_nt, raster_group(M, 2 * F, K),
                                                                    kind, stream);
}

}  // namespace

// =========================================================================
// extern "C"
// =========================================================================

extern "C" {

const char* coda_status_string(coda_status_t s) {
  switch (s) {
    case CODA_OK: return "CODA_OK";
    case CODA_ERR_NULL: return "CODA_ERR_NULL: a required pointer is NULL";
    case CODA_ERR_SHAPE: return "CODA_ERR_SHAPE: invalid size (sizes must be > 0 and multiples of 8; M >= 0)";
    case CODA_ERR_ALIGN: return "CODA_ERR_ALIGN: a pointer is not 16-byte aligned";
    case CODA_ERR_WORKSPACE: return "CODA_ERR_WORKSPACE: workspace missing or too small";
    case CODA_ERR_DEVICE: return "CODA_ERR_DEVICE: no CUDA device or not compute capability 10.0";
    case CODA_ERR_LAUNCH: return "CODA_ERR_LAUNCH: a CUDA runtime call failed";
    case CODA_ERR_DEVICE_TIMEOUT: return "CODA_ERR_DEVICE_TIMEOUT: a kernel gave up on a bounded wait";
    case CODA_ERR_INTERNAL: return "CODA_ERR_INTERNAL: internal failure (tensor map encoding)";
  }
  return "CODA_ERR_UNKNOWN";
}

int coda_version(void) { return kVersion; }

int64_t coda_partial_tile_width(void) { return kPartialTile; }

int64_t coda_partial_cols(int64_t N) { return N <= 0 ? -1 : (N + kPartialTile - 1) / kPartialTile; }

coda_status_t coda_set_wait_limit_ns(int64_t ns) {
  if (ns <= 0) return CODA_ERR_SHAPE;
  g_wait_ns = ns;
  return CODA_OK;
}

coda_status_t coda_poll_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return CODA_ERR_LAUNCH;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_coda_status, sizeof(int)) != cudaSuccess) return CODA_ERR_LAUNCH;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_coda_status, &zero, sizeof(int)) != cudaSuccess) return CODA_ERR_LAUNCH;
    return CODA_ERR_DEVICE_TIMEOUT;
  }
  return CODA_OK;
}

// ------------------------------------------------------------------ forward

coda_status_t coda_gemm_res_partialrms(const uint16_t* x, const uint16_t* W, const uint16_t* res,
                                       const uint16_t* gamma, uint16_t* h_out, uint16_t* hg_out, float* partial,
                                       int64_t M, int64_t N, int64_t K, void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && dim_ok(N) && dim_ok(K), CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(x && W, CODA_ERR_NULL);
  CODA_CHECK(h_out || hg_out || partial, CODA_ERR_NULL);
  CODA_CHECK(!hg_out || gamma, CODA_ERR_NULL);
  CODA_CHECK(al16(x) && al16(W) && al16(res) && al16(gamma) && al16(h_out) && al16(hg_out) && al16(partial),
             CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  using Epi = EpiLoadStore2<0>;
  GemmParams<Epi> p{};
  bool ok = map_a(&p.tmA, x, false, M, K) && map_b(&p.tmB, W, true, N, K, N, 128);
  if (h_out) ok = ok && map_out_bf16(&p.ep.tmOut1, h_out, M, N, N);
  if (hg_out) ok = ok && map_out_bf16(&p.ep.tmOut2, hg_out, M, N, N);
  if (!ok) return CODA_ERR_INTERNAL;
  p.ep.in = reinterpret_cast<const __nv_bfloat16*>(res);
  p.ep.gamma = reinterpret_cast<const __nv_bfloat16*>(gamma);
  p.ep.r = nullptr;
  p.ep.partial = partial;
  p.ep.has_out1 = h_out != nullptr;
  p.ep.has_out2 = hg_out != nullptr;
  const int n_nt = static_cast<int>((N + 255) / 256);
  return run_gemm<256, pair_stages<Epi>(), false, true, true, Epi>(dev, info, p, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), n_nt,
      raster_group(M, N, K), kKindResPartial, static_cast<cudaStream_t>(stream));
}

coda_status_t coda_rms_reduce(const float* partial, int64_t M, int64_t T, int64_t N, float eps, float* r_out,
                              void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && T > 0 && N > 0 && T <= 1 << 20 && eps >= 0.f, CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(partial && r_out, CODA_ERR_NULL);
  CODA_CHECK(al16(partial) && al16(r_out), CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  coda_status_t st = current_device(&dev, &info);
  if (st != CODA_OK) return st;
  const int threads = 256;
  const int blocks = static_cast<int>((M + threads - 1) / threads);
  rms_reduce_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
      partial, static_cast<int>(M), static_cast<int>(T), 1.0f / static_cast<float>(N), eps, r_out);
  return cudaGetLastError() == cudaSuccess ? CODA_OK : CODA_ERR_LAUNCH;
}

coda_status_t coda_gemm_rowscale(const uint16_t* A, const uint16_t* W, const float* r, uint16_t* out, int64_t M,
                                 int64_t N, int64_t K, void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && dim_ok(N) && dim_ok(K), CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(A && W && out, CODA_ERR_NULL);
  CODA_CHECK(al16(A) && al16(W) && al16(r) && al16(out), CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  using Epi = EpiRowScale;
  GemmParams<Epi> p{};
  if (!(map_a(&p.tmA, A, false, M, K) && map_b(&p.tmB, W, true, N, K, N, 128) &&
        map_out_bf16(&p.ep.tmOut, out, M, N, N)))
    return CODA_ERR_INTERNAL;
  p.ep.r = r;
  const int n_nt = static_cast<int>((N + 255) / 256);
  return run_gemm<256, pair_stages<Epi>(), false, true, true, Epi>(dev, info, p, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), n_nt,
      raster_group(M, N, K), kKindRowScale, static_cast<cudaStream_t>(stream));
}

size_t coda_rmsnorm_block_workspace_size(int64_t M) {
  if (M < 0) return 0;
  return align256(static_cast<size_t>((M + 255) / 256) * 4);
}

coda_status_t coda_rmsnorm_block(const uint16_t* x, const uint16_t* res, const uint16_t* W1, const uint16_t* W2,
                                 const uint16_t* gamma, float eps, uint16_t* h_out, uint16_t* hg_out,
                                 float* partial_out, float* r_out, uint16_t* out, void* ws, size_t ws_bytes,
                                 int64_t M, int64_t K, int64_t N, int64_t N2, void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && dim_ok(K) && dim_ok(N) && dim_ok(N2) && eps >= 0.f,
             CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(x && W1 && W2 && gamma && h_out && hg_out && partial_out && out, CODA_ERR_NULL);
  CODA_CHECK(al16(x) && al16(res) && al16(W1) && al16(W2) && al16(gamma) && al16(h_out) && al16(hg_out) &&
                 al16(partial_out) && al16(r_out) && al16(out) && al16(ws),
             CODA_ERR_ALIGN);
  CODA_CHECK(ws != nullptr && ws_bytes >= coda_rmsnorm_block_workspace_size(M), CODA_ERR_WORKSPACE);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  constexpr int kStages = 6;
  auto kern = coda_block_kernel<kStages>;
  constexpr int smem = BlockSmem<kStages>::kBytes;
  static_assert(smem <= 232448, "the block kernel's shared memory exceeds one SM's opt-in limit");
  KernelCache& kc = g_kcache[dev][kKindBlock];
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!kc.attr) {
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return CODA_ERR_LAUNCH;
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * (info->sms / 2), 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = info->sms / 2;
      }
      kc.max_clusters = n;
      kc.attr = true;
    }
  }
  BlockParams p{};
  bool ok = map_a(&p.tmA1, x, false, M, K) && map_b(&p.tmB1, W1, true, N, K, N, 128) &&
            map_a(&p.tmA2, hg_out, false, M, N) && map_b(&p.tmB2, W2, true, N2, N, N2, 128) &&
            map_out_bf16(&p.ep1.tmOut1, h_out, M, N, N) && map_out_bf16(&p.ep1.tmOut2, hg_out, M, N, N) &&
            map_out_bf16(&p.ep2.tmOut, out, M, N2, N2);
  if (!ok) return CODA_ERR_INTERNAL;
  p.ep1.in = reinterpret_cast<const __nv_bfloat16*>(res);
  p.ep1.gamma = reinterpret_cast<const __nv_bfloat16*>(gamma);
  p.ep1.r = nullptr;
  p.ep1.partial = partial_out;
  p.ep1.has_out1 = 1;
  p.ep1.has_out2 = 1;
  p.ep2.r = nullptr;
  p.ep2.partial = partial_out;
  p.ep2.T = static_cast<int>(coda_partial_cols(N));
  p.ep2.inv_n = 1.0f / static_cast<float>(N);
  p.ep2.eps = eps;
  p.ep2.r_out = r_out;
  p.ready = static_cast<int*>(ws);
  p.M = static_cast<int>(M);
  p.K1 = static_cast<int>(K);
  p.N1 = static_cast<int>(N);
  p.N2 = static_cast<int>(N2);
  p.n_mt = static_cast<int>((M + 255) / 256);
  p.n_nt1 = static_cast<int>((N + 255) / 256);
  p.n_nt2 = static_cast<int>((N2 + 255) / 256);
  p.n1 = p.n_mt * p.n_nt1;
  p.n2 = p.n_mt * p.n_nt2;
  // second-GEMM tiles in groups of row blocks whose hg takes 16 MiB (16 row
  // blocks at hidden 2048): 451 against 462 us at the 1B block tail with all
  // row blocks of a column block in turn, whose first tiles wait for the
  // first GEMM's last wave
  {
    const int64_t g2 = (int64_t(16) << 20) / (2 * int64_t(kBM) * N * 2);
    p.group2 = static_cast<int>(g2 < 1 ? 1 : (g2 > p.n_mt ? p.n_mt : g2));
  }
  p.ready_target = p.n_nt1 * 2 * kEpiWarps;
  p.wait_ns = static_cast<uint64_t>(g_wait_ns);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, static_cast<size_t>(p.n_mt) * 4, s) != cudaSuccess) return CODA_ERR_LAUNCH;
  // as in run_gemm: a last partial wave on at most half of the pairs runs as
  // half tiles (of the second GEMM, whose tiles come last)
  p.nsplit = 0;
  {
    const int last = (p.n1 + p.n2) % kc.max_clusters;
    if (last > 0 && 2 * last <= kc.max_clusters) p.nsplit = last < p.n2 ? last : p.n2;
  }
  const int total = p.n1 + p.n2 + p.nsplit;
  const int clusters = total < kc.max_clusters ? total : kc.max_clusters;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return CODA_ERR_LAUNCH;
  return cudaGetLastError() == cudaSuccess ? CODA_OK : CODA_ERR_LAUNCH;
}

coda_status_t coda_gemm_rowscale_partial(const uint16_t* A, const uint16_t* W, const float* partial, int64_t T,
                                         int64_t N_norm, float eps, float* r_out, uint16_t* out, int64_t M,
                                         int64_t N, int64_t K, void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && dim_ok(N) && dim_ok(K) && T > 0 && T <= 1 << 20 && N_norm > 0 &&
                 eps >= 0.f,
             CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(A && W && partial && out, CODA_ERR_NULL);
  CODA_CHECK(al16(A) && al16(W) && al16(partial) && al16(r_out) && al16(out), CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  using Epi = EpiRowScale;
  GemmParams<Epi> p{};
  if (!(map_a(&p.tmA, A, false, M, K) && map_b(&p.tmB, W, true, N, K, N, 128) &&
        map_out_bf16(&p.ep.tmOut, out, M, N, N)))
    return CODA_ERR_INTERNAL;
  p.ep.r = nullptr;
  p.ep.partial = partial;
  p.ep.T = static_cast<int>(T);
  p.ep.inv_n = 1.0f / static_cast<float>(N_norm);
  p.ep.eps = eps;
  p.ep.r_out = r_out;
  const int n_nt = static_cast<int>((N + 255) / 256);
  return run_gemm<256, pair_stages<Epi>(), false, true, true, Epi>(dev, info, p, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), n_nt,
      raster_group(M, N, K), kKindRowScale, static_cast<cudaStream_t>(stream));
}

coda_status_t coda_gemm_swiglu(const uint16_t* A, const uint16_t* W_gu, const float* r, uint16_t* act_out,
                               uint16_t* gateup_save, int64_t M, int64_t F, int64_t K, void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && dim_ok(F) && dim_ok(K), CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(A && W_gu && act_out, CODA_ERR_NULL);
  CODA_CHECK(al16(A) && al16(W_gu) && al16(r) && al16(act_out) && al16(gateup_save), CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (gateup_save)
    return run_swiglu<EpiSwiGLU>(dev, info, A, W_gu, r, act_out, gateup_save, M, F, K, kKindSwiGLU, s);
  return run_swiglu<EpiSwiGLUAct>(dev, info, A, W_gu, r, act_out, nullptr, M, F, K, kKindSwiGLUAct, s);
}

coda_status_t coda_gemm_qkv_rope(const uint16_t* x, const uint16_t* W_qkv, const int32_t* positions, uint16_t* out,
                                 int64_t M, int64_t N, int64_t K, int64_t head_dim, int64_t rope_cols, float theta,
                                 void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && dim_ok(N) && dim_ok(K) && (head_dim == 64 || head_dim == 128) &&
                 N % head_dim == 0 && rope_cols >= 0 && rope_cols <= N && rope_cols % head_dim == 0 &&
                 theta > 1.0f,
             CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(x && W_qkv && positions && out, CODA_ERR_NULL);
  CODA_CHECK(al16(x) && al16(W_qkv) && al16(positions) && al16(out), CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  using Epi = EpiRope;
  GemmParams<Epi> p{};
  if (!(map_a(&p.tmA, x, false, M, K) && map_b(&p.tmB, W_qkv, true, N, K, N, 128) &&
        map_out_bf16(&p.ep.tmOut, out, M, N, N)))
    return CODA_ERR_INTERNAL;
  p.ep.positions = positions;
  p.ep.head_dim = static_cast<int>(head_dim);
  p.ep.rope_cols = static_cast<int>(rope_cols);
  // The angle of frequency i in turns, theta^(-2i/head_dim) / (2 pi) < 1, as a
  // 64-bit fraction (ldexp by 64 stays below 2^64; the conversion drops less
  // than 2^-64 turn, which a position below 2^31 grows to under 2^-33 turn).
  for (int i = 0; i < head_dim / 2; ++i)
    p.ep.turn_fx[i] = static_cast<uint64_t>(
        std::ldexp(std::pow(static_cast<double>(theta), -2.0 * i / static_cast<double>(head_dim)) / (2.0 * M_PI), 64));
  return run_gemm<256, pair_stages<Epi>(), false, true, true, Epi>(
      dev, info, p, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), static_cast<int>((N + 255) / 256),
      raster_group(M, N, K), kKindRope, static_cast<cudaStream_t>(stream));
}

coda_status_t coda_gemm_swiglu_bwd(const uint16_t* d_out, const uint16_t* W_down, const uint16_t* gateup,
                                   uint16_t* d_gateup_out, int64_t M, int64_t F, int64_t N, void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && dim_ok(F) && dim_ok(N), CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(d_out && W_down && gateup && d_gateup_out, CODA_ERR_NULL);
  CODA_CHECK(al16(d_out) && al16(W_down) && al16(gateup) && al16(d_gateup_out), CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  using Epi = EpiSwiGLUBwd;
  GemmParams<Epi> p{};
  // d_act = d_out W_down^T: W_down [F, N] read as [F rows of length N] (K-major), GEMM K = N.
  if (!(map_a(&p.tmA, d_out, false, M, N) && map_b(&p.tmB, W_down, false, F, N, N, 128) &&
        map_out_bf16(&p.ep.tmG, gateup, M, F, 2 * F) && map_out_bf16(&p.ep.tmU, gateup + F, M, F, 2 * F) &&
        map_out_bf16(&p.ep.tmDG, d_gateup_out, M, F, 2 * F) &&
        map_out_bf16(&p.ep.tmDU, d_gateup_out + F, M, F, 2 * F)))
    return CODA_ERR_INTERNAL;
  const int n_nt = static_cast<int>((F + 255) / 256);
  return run_gemm<256, pair_stages<Epi>(), false, false, true, Epi>(
      dev, info, p, static_cast<int>(M), static_cast<int>(F), static_cast<int>(N), n_nt, raster_group(M, F, N),
      kKindSwiGLUBwd, static_cast<cudaStream_t>(stream));
}

size_t coda_lmhead_ce_workspace_size(int64_t M, int64_t V) {
  if (M < 0 || V <= 0) return 0;
  return ce_ws_bytes(M, V);
}

coda_status_t coda_lmhead_ce(const uint16_t* H, const uint16_t* W, const int64_t* labels, const float* r,
                             float* loss_out, float* lse_out, float* mean_out, void* ws, size_t ws_bytes,
                             int64_t M, int64_t V, int64_t K, void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && dim_ok(V) && dim_ok(K), CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(H && W && labels && loss_out && lse_out, CODA_ERR_NULL);
  CODA_CHECK(al16(H) && al16(W) && al16(labels) && al16(r) && al16(loss_out) && al16(lse_out) && al16(ws),
             CODA_ERR_ALIGN);
  CODA_CHECK(ws != nullptr && ws_bytes >= ce_ws_bytes(M, V), CODA_ERR_WORKSPACE);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  using Epi = EpiCE;
  GemmParams<Epi> p{};
  if (!(map_a(&p.tmA, H, false, M, K) && map_b(&p.tmB, W, true, V, K, V, 128))) return CODA_ERR_INTERNAL;
  const int n_nt = static_cast<int>((V + 255) / 256);
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.ep.ws_m = reinterpret_cast<float*>(w);
  p.ep.ws_s = reinterpret_cast<float*>(w + align256(static_cast<size_t>(n_nt) * M * 4));
  p.ep.zlab = reinterpret_cast<float*>(w + 2 * align256(static_cast<size_t>(n_nt) * M * 4));
  p.ep.labels = labels;
  p.ep.r = r;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  coda_status_t st = run_gemm<256, pair_stages<Epi>(), false, true, true, Epi>(dev, info, p, static_cast<int>(M), static_cast<int>(V),
                                                        static_cast<int>(K), n_nt, raster_group(M, V, K), kKindCE, s);
  if (st != CODA_OK) return st;
  ce_combine_kernel<<<static_cast<int>((M + 31) / 32), 32 * kCombWarps, 0, s>>>(
      p.ep.ws_m, p.ep.ws_s, p.ep.zlab, labels, static_cast<int>(M), n_nt, V, lse_out, loss_out);
  if (cudaGetLastError() != cudaSuccess) return CODA_ERR_LAUNCH;
  if (mean_out) {
    mean_kernel<<<1, 1024, 0, s>>>(loss_out, static_cast<int>(M), mean_out);
    if (cudaGetLastError() != cudaSuccess) return CODA_ERR_LAUNCH;
  }
  return CODA_OK;
}

// ----------------------------------------------------------------- backward

size_t coda_lmhead_ce_bwd_workspace_size(int64_t M, int64_t V) {
  if (M < 0 || V <= 0) return 0;
  const int64_t vc = V < kCEBwdChunk ? V : kCEBwdChunk;
  const size_t nb = static_cast<size_t>((V + kLabelTile - 1) / kLabelTile);
  return align256(static_cast<size_t>(M) * static_cast<size_t>(vc) * 2)  // G chunk (bf16)
         + align256(static_cast<size_t>(M) * 4)                           // label residuals
         + 2 * align256(nb * 4) + align256((nb + 1) * 4)                  // bucket counts, cursors, offsets
         + 2 * align256(static_cast<size_t>(M) * 8);                      // (label, row) entries, two copies
}

coda_status_t coda_lmhead_ce_bwd(const uint16_t* H, const uint16_t* W, const int64_t* labels, const float* lse,
                                 const float* d_loss, const float* r, float* dH_out, float* dW_out, void* ws,
                                 size_t ws_bytes, int64_t M, int64_t V, int64_t K, void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && dim_ok(V) && dim_ok(K), CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(H && W && labels && lse && dH_out && dW_out, CODA_ERR_NULL);
  CODA_CHECK(al16(H) && al16(W) && al16(labels) && al16(lse) && al16(d_loss) && al16(r) && al16(dH_out) &&
                 al16(dW_out) && al16(ws),
             CODA_ERR_ALIGN);
  CODA_CHECK(ws != nullptr && ws_bytes >= coda_lmhead_ce_bwd_workspace_size(M, V), CODA_ERR_WORKSPACE);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t vmax = V < kCEBwdChunk ? V : kCEBwdChunk;
  const int nbk = static_cast<int>((V + kLabelTile - 1) / kLabelTile);
  uint8_t* wp = static_cast<uint8_t*>(ws);
  uint16_t* G = reinterpret_cast<uint16_t*>(wp);
  wp += align256(static_cast<size_t>(M) * vmax * 2);
  float* resid = reinterpret_cast<float*>(wp);
  wp += align256(static_cast<size_t>(M) * 4);
  int* counts = reinterpret_cast<int*>(wp);
  wp += align256(static_cast<size_t>(nbk) * 4);
  int* cursor = reinterpret_cast<int*>(wp);
  wp += align256(static_cast<size_t>(nbk) * 4);
  int* start = reinterpret_cast<int*>(wp);
  wp += align256(static_cast<size_t>(nbk + 1) * 4);
  int2* unsorted = reinterpret_cast<int2*>(wp);
  wp += align256(static_cast<size_t>(M) * 8);
  int2* entries = reinterpret_cast<int2*>(wp);
  {
    // rows bucketed by the 256-column vocabulary tile of their label, sorted by (label, row)
    const int mi = static_cast<int>(M);
    const int g = (mi + 255) / 256;
    if (cudaMemsetAsync(counts, 0, static_cast<size_t>(nbk) * 4, s) != cudaSuccess) return CODA_ERR_LAUNCH;
    ce_label_count_kernel<<<g, 256, 0, s>>>(labels, mi, V, counts);
    ce_label_scan_kernel<<<1, 1024, 0, s>>>(counts, nbk, start, cursor);
    ce_label_fill_kernel<<<g, 256, 0, s>>>(labels, mi, V, cursor, unsorted);
    ce_label_sort_kernel<<<g, 256, 0, s>>>(unsorted, start, nbk, entries);
    if (cudaGetLastError() != cudaSuccess) return CODA_ERR_LAUNCH;
  }
  for (int64_t c0 = 0; c0 < V; c0 += kCEBwdChunk) {
    const int64_t vc = (V - c0) < kCEBwdChunk ? (V - c0) : kCEBwdChunk;
    {
      // G = d (exp(z - lse) - onehot) for z = r (H W[:, c0:c0+vc]), bf16 [M, vc]
      using Epi = EpiCEGrad;
      GemmParams<Epi> p{};
      if (!(map_a(&p.tmA, H, false, M, K) && map_b(&p.tmB, W + c0, true, vc, K, V, 128) &&
            map_out_bf16(&p.ep.tmG, G, M, vc, vc)))
        return CODA_ERR_INTERNAL;
      p.ep.labels = labels;
      p.ep.lse = lse;
      p.ep.d_loss = d_loss;
      p.ep.r = r;
      p.ep.scale = 1.0f / static_cast<float>(M);
      p.ep.col_offset = c0;
      p.ep.resid = resid;
      if (c0 > 0) {
        // the previous chunk's label entries of dH, added before this chunk's first tile
        const int64_t p0 = c0 - kCEBwdChunk;
        p.ep.fix_entries = entries;
        p.ep.fix_start = start;
        p.ep.fix_b0 = static_cast<int>(p0 / kLabelTile);
        p.ep.fix_b1 = static_cast<int>((c0 + kLabelTile - 1) / kLabelTile);
        p.ep.fix_W = reinterpret_cast<const __nv_bfloat16*>(W);
        p.ep.fix_V = V;
        p.ep.fix_K = static_cast<int>(K);
        p.ep.fix_dH = dH_out;
      }
      const coda_status_t st = run_gemm<256, pair_stages<Epi>(), false, true, true, Epi>(
          dev, info, p, static_cast<int>(M), static_cast<int>(vc), static_cast<int>(K),
          static_cast<int>((vc + 255) / 256), raster_group(M, vc, K), kKindCEGrad, s);
      if (st != CODA_OK) return st;
    }
    {
      // dW[:, chunk] = H^T G (problem 0: GEMM K = tokens, the longer tiles;
      // A = H read transposed (MN-major), B = G (MN-major)) and
      // dH (+)= G W[:, chunk]^T (problem 1: GEMM K = vc; B = the chunk of W
      // read as [K rows of length vc] (K-major)) in one grouped launch.
      GroupedParams<EpiStoreF32, EpiStoreF32> p{};
      if (!(map_a(&p.tmA[0], H, true, K, M) && map_b(&p.tmB[0], G, true, vc, M, vc, 128) &&
            map_out_f32_ld(&p.ep0.tmOut, dW_out + c0, K, vc, V) && map_a(&p.tmA[1], G, false, M, vc) &&
            map_b(&p.tmB[1], W + c0, false, K, vc, V, 128) && map_out_f32(&p.ep1.tmOut, dH_out, M, K)))
        return CODA_ERR_INTERNAL;
      p.ep0.add_to_out = 0;
      p.ep0.fix_resid = resid;
      p.ep0.fix_col0 = c0;
      p.ep0.fix_start = start;
      p.ep0.fix_entries = entries;
      p.ep0.fix_H = reinterpret_cast<const __nv_bfloat16*>(H);
      p.ep0.fix_tile0 = static_cast<int>(c0 / kLabelTile);
      p.ep1.add_to_out = c0 == 0 ? 0 : 1;  // dH: the first chunk stores, the others add in L2
      const GroupedProblem pb[2] = {
          {static_cast<int>(K), static_cast<int>(vc), static_cast<int>(M), raster_group(K, vc, M), true, true},
          {static_cast<int>(M), static_cast<int>(K), static_cast<int>(vc), raster_group(M, K, vc), false, false}};
      const coda_status_t st = run_grouped(dev, info, p, pb, kKindGroupedCE, s);
      if (st != CODA_OK) return st;
    }
    if (c0 + vc >= V) {
      // the last chunk's label entries of dH (every earlier chunk's are added
      // by the next chunk's gradient GEMM before its first tile)
      ce_label_dh_fix_kernel<<<info->sms * 4, 256, 0, s>>>(
          entries, start, static_cast<int>(c0 / kLabelTile),
          static_cast<int>((c0 + vc + kLabelTile - 1) / kLabelTile), resid, reinterpret_cast<const __nv_bfloat16*>(W),
          V, static_cast<int>(K), dH_out);
      if (cudaGetLastError() != cudaSuccess) return CODA_ERR_LAUNCH;
    }
  }
  return CODA_OK;
}

coda_status_t coda_loss_stats(const float* loss, int64_t M, float* stats_out, void* stream) {
  CODA_CHECK(M > 0 && M < (int64_t(1) << 24), CODA_ERR_SHAPE);  // the count is exact in fp32
  CODA_CHECK(loss && stats_out, CODA_ERR_NULL);
  CODA_CHECK(al16(loss) && al16(stats_out), CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  loss_stats_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(loss, static_cast<int>(M), stats_out);
  return cudaGetLastError() == cudaSuccess ? CODA_OK : CODA_ERR_LAUNCH;
}

coda_status_t coda_ce_global_finish(const float* stats, int64_t M, float* mean_out, float* d_loss_out,
                                    void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31), CODA_ERR_SHAPE);
  CODA_CHECK(stats && (mean_out || d_loss_out), CODA_ERR_NULL);
  CODA_CHECK(al16(stats) && al16(mean_out) && al16(d_loss_out), CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  const int grid = d_loss_out != nullptr && M > 256 ? static_cast<int>((M + 255) / 256 < info->sms ? (M + 255) / 256
                                                                                                    : info->sms)
                                                      : 1;
  ce_global_finish_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(stats, static_cast<int>(M), mean_out,
                                                                               d_loss_out);
  return cudaGetLastError() == cudaSuccess ? CODA_OK : CODA_ERR_LAUNCH;
}

size_t coda_gemm_rowscale_bwd_workspace_size(int64_t M, int64_t N) {
  if (M < 0 || N <= 0) return 0;
  return align256(static_cast<size_t>(M) * N * 2);
}

coda_status_t coda_gemm_rowscale_bwd(const uint16_t* dOut, const uint16_t* hg, const uint16_t* W2, const float* r,
                                     float* d_hg_out, float* dW2_out, float* pdr_out, void* ws, size_t ws_bytes,
                                     int64_t M, int64_t N, int64_t N2, void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && dim_ok(N) && dim_ok(N2), CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(dOut && hg && W2 && r && d_hg_out && dW2_out && pdr_out, CODA_ERR_NULL);
  CODA_CHECK(al16(dOut) && al16(hg) && al16(W2) && al16(r) && al16(d_hg_out) && al16(dW2_out) && al16(pdr_out) &&
                 al16(ws),
             CODA_ERR_ALIGN);
  CODA_CHECK(ws != nullptr && ws_bytes >= coda_gemm_rowscale_bwd_workspace_size(M, N), CODA_ERR_WORKSPACE);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  uint16_t* y = static_cast<uint16_t*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  {
    // P = dOut W2^T with the block-local epilogue (d_hg, y, pdr).
    using Epi = EpiLoadStore2<1>;
    GemmParams<Epi> p{};
    if (!(map_a(&p.tmA, dOut, false, M, N2) && map_b(&p.tmB, W2, false, N, N2, N2, 128) &&
          map_b(&p.tmBh, W2, false, N, N2, N2, 64) && map_out_bf16(&p.ep.tmOut1, y, M, N, N) &&
          map_out_f32(&p.ep.tmOut2, d_hg_out, M, N)))
      return CODA_ERR_INTERNAL;
    p.has_bh = 1;
    p.ep.in = reinterpret_cast<const __nv_bfloat16*>(hg);
    p.ep.gamma = nullptr;
    p.ep.r = r;
    p.ep.partial = pdr_out;
    p.ep.has_out1 = 1;
    p.ep.has_out2 = 1;
    // a split by k-blocks adds into d_hg [M, N] and pdr [T, M]
    const ZeroPlan zp[2] = {
        {d_hg_out, static_cast<size_t>(N) * 4, 4, M, N, 256, 256, false},
        {pdr_out, static_cast<size_t>(M) * 4, 4, coda_partial_cols(N), M, 2, 256, true}};
    coda_status_t st = run_gemm<256, pair_stages<Epi>(), false, false, true, Epi>(dev, info, p, static_cast<int>(M), static_cast<int>(N),
                                                           static_cast<int>(N2), static_cast<int>((N + 255) / 256),
                                                           raster_group(M, N, N2), kKindBwdP, s, zp, 2);
    if (st != CODA_OK) return st;
  }
  {
    // dW2 = y^T dOut: A = y read transposed (MN-major), B = dOut (MN-major), K = tokens.
    using Epi = EpiStoreF32;
    GemmParams<Epi> p{};
    if (!(map_a(&p.tmA, y, true, N, M) && map_b(&p.tmB, dOut, true, N2, M, N2, 128) &&
          map_out_f32(&p.ep.tmOut, dW2_out, N, N2)))
      return CODA_ERR_INTERNAL;
    const ZeroPlan zp = {dW2_out, static_cast<size_t>(N2) * 4, 4, N, N2, 256, 256, false};
    return run_gemm<256, pair_stages<Epi>(), true, true, true, Epi>(dev, info, p, static_cast<int>(N), static_cast<int>(N2), static_cast<int>(M), static_cast<int>((N2 + 255) / 256),
      raster_group(N, N2, M), kKindF32MN, s, &zp, 1);
  }
}

size_t coda_rms_reduce_bwd_workspace_size(int64_t M, int64_t N) {
  if (M < 0 || N <= 0) return 0;
  return align256(static_cast<size_t>((M + kBwdRows - 1) / kBwdRows) * N * 4);
}

coda_status_t coda_rms_reduce_bwd(const float* pdr, const float* r, const float* d_hg, const uint16_t* h,
                                  const uint16_t* gamma, uint16_t* dh_out, float* dgamma_out, void* ws,
                                  size_t ws_bytes, int64_t M, int64_t T, int64_t N, void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && T > 0 && T <= 1 << 20 && dim_ok(N), CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(pdr && r && d_hg && h && gamma && dh_out && dgamma_out, CODA_ERR_NULL);
  CODA_CHECK(al16(pdr) && al16(r) && al16(d_hg) && al16(h) && al16(gamma) && al16(dh_out) && al16(dgamma_out) &&
                 al16(ws),
             CODA_ERR_ALIGN);
  CODA_CHECK(ws != nullptr && ws_bytes >= coda_rms_reduce_bwd_workspace_size(M, N), CODA_ERR_WORKSPACE);
  int dev = 0;
  DevInfo* info = nullptr;
  coda_status_t st = current_device(&dev, &info);
  if (st != CODA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int nblk = static_cast<int>((M + kBwdRows - 1) / kBwdRows);
  float* part = static_cast<float*>(ws);
  rms_reduce_bwd_kernel<<<nblk, kBwdThreads, 0, s>>>(
      pdr, r, d_hg, reinterpret_cast<const __nv_bfloat16*>(h),
      reinterpret_cast<const __nv_bfloat16*>(gamma), reinterpret_cast<__nv_bfloat16*>(dh_out), part,
      static_cast<int>(M), static_cast<int>(T), static_cast<int>(N));
  if (cudaGetLastError() != cudaSuccess) return CODA_ERR_LAUNCH;
  dgamma_final_kernel<<<static_cast<int>((N + kDgCols - 1) / kDgCols), kDgCols * kDgGroups, 0, s>>>(part, nblk, static_cast<int>(N), dgamma_out);
  return cudaGetLastError() == cudaSuccess ? CODA_OK : CODA_ERR_LAUNCH;
}

coda_status_t coda_gemm_res_partialrms_bwd(const uint16_t* dh, const uint16_t* x, const uint16_t* W1,
                                           uint16_t* dx_out, float* dW1_out, int64_t M, int64_t N, int64_t K,
                                           void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && dim_ok(N) && dim_ok(K), CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(dh && x && W1, CODA_ERR_NULL);
  CODA_CHECK(dx_out || dW1_out, CODA_ERR_NULL);
  CODA_CHECK(al16(dh) && al16(x) && al16(W1) && al16(dx_out) && al16(dW1_out), CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dx_out && dW1_out && M >= N) {
    // Both products in one grouped launch, dW1 (GEMM K = M, the longer tiles)
    // first.  Taken only when dW1 is the longer one: with dx longer (N > M,
    // as in the SwiGLU MLP's d_y = d_gu W_gu^T with N = 16384) the two
    // problems' operands (over 200 MB) compete for L2 and the grouped launch
    // measured 8 % slower than two launches (0.82 against 0.76 ms).
    GroupedParams<EpiStoreF32, EpiRowScale> p{};
    if (!(map_a(&p.tmA[0], x, true, K, M) && map_b(&p.tmB[0], dh, true, N, M, N, 128) &&
          map_a(&p.tmA[1], dh, false, M, N) && map_b(&p.tmB[1], W1, false, K, N, N, 128) &&
          map_out_f32(&p.ep0.tmOut, dW1_out, K, N) && map_out_bf16(&p.ep1.tmOut, dx_out, M, K, K)))
      return CODA_ERR_INTERNAL;
    const GroupedProblem pb[2] = {
        {static_cast<int>(K), static_cast<int>(N), static_cast<int>(M), raster_group(K, N, M), true, true},
        {static_cast<int>(M), static_cast<int>(K), static_cast<int>(N), raster_group(M, K, N), false, false}};
    return run_grouped(dev, info, p, pb, kKindGroupedWX, s);
  }
  if (dx_out) {
    // dx = dh W1^T: B = W1 read as [K rows of length N] (K-major), GEMM K = N.
    using Epi = EpiRowScale;
    GemmParams<Epi> p{};
    if (!(map_a(&p.tmA, dh, false, M, N) && map_b(&p.tmB, W1, false, K, N, N, 128) &&
          map_b(&p.tmBh, W1, false, K, N, N, 64) && map_out_bf16(&p.ep.tmOut, dx_out, M, K, K)))
      return CODA_ERR_INTERNAL;
    p.has_bh = 1;
    p.ep.r = nullptr;
    coda_status_t st = run_gemm<256, pair_stages<Epi>(), false, false, true, Epi>(dev, info, p, static_cast<int>(M), static_cast<int>(K),
                                                           static_cast<int>(N), static_cast<int>((K + 255) / 256),
                                                           raster_group(M, K, N), kKindRowScaleKK, s);
    if (st != CODA_OK) return st;
  }
  if (dW1_out) {
    // dW1 = x^T dh: A = x read transposed (MN-major), B = dh (MN-major), K = tokens.
    using Epi = EpiStoreF32;
    GemmParams<Epi> p{};
    if (!(map_a(&p.tmA, x, true, K, M) && map_b(&p.tmB, dh, true, N, M, N, 128) &&
          map_out_f32(&p.ep.tmOut, dW1_out, K, N)))
      return CODA_ERR_INTERNAL;
    const ZeroPlan zp = {dW1_out, static_cast<size_t>(N) * 4, 4, K, N, 256, 256, false};
    return run_gemm<256, pair_stages<Epi>(), true, true, true, Epi>(dev, info, p, static_cast<int>(K), static_cast<int>(N), static_cast<int>(M), static_cast<int>((N + 255) / 256),
      raster_group(K, N, M), kKindF32MN, s, &zp, 1);
  }
  return CODA_OK;
}

// --------------------------------------------------- unfused comparison chain

coda_status_t coda_unfused_add(const uint16_t* a, const uint16_t* b, uint16_t* out, int64_t n, void* stream) {
  CODA_CHECK(a && b && out, CODA_ERR_NULL);
  CODA_CHECK(n >= 0 && n % 8 == 0, CODA_ERR_SHAPE);
  CODA_CHECK(al16(a) && al16(b) && al16(out), CODA_ERR_ALIGN);
  if (n == 0) return CODA_OK;
  int dev = 0;
  DevInfo* info = nullptr;
  coda_status_t st = current_device(&dev, &info);
  if (st != CODA_OK) return st;
  const size_t n8 = static_cast<size_t>(n / 8);
  const int threads = 256;
  size_t blocks = (n8 + threads - 1) / threads;
  const size_t cap = static_cast<size_t>(info->sms) * 8;
  if (blocks > cap) blocks = cap;
  add_bf16_kernel<<<static_cast<int>(blocks), threads, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(a), reinterpret_cast<const __nv_bfloat16*>(b),
      reinterpret_cast<__nv_bfloat16*>(out), n8);
  return cudaGetLastError() == cudaSuccess ? CODA_OK : CODA_ERR_LAUNCH;
}

coda_status_t coda_unfused_rmsnorm(const uint16_t* h, const uint16_t* gamma, float eps, uint16_t* y_out,
                                   float* r_out, int64_t M, int64_t N, void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && dim_ok(N) && eps >= 0.f, CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(h && gamma && y_out, CODA_ERR_NULL);
  CODA_CHECK(al16(h) && al16(gamma) && al16(y_out) && al16(r_out), CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  coda_status_t st = current_device(&dev, &info);
  if (st != CODA_OK) return st;
  rmsnorm_kernel<<<static_cast<int>(M), kNormThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(h), reinterpret_cast<const __nv_bfloat16*>(gamma), eps,
      reinterpret_cast<__nv_bfloat16*>(y_out), r_out, static_cast<int>(N));
  return cudaGetLastError() == cudaSuccess ? CODA_OK : CODA_ERR_LAUNCH;
}

// ------------------------------------------------------------------- testing

coda_status_t coda_selftest_bounded_wait(int64_t limit_ns, int* gave_up_dev, void* stream) {
  CODA_CHECK(gave_up_dev, CODA_ERR_NULL);
  CODA_CHECK(limit_ns > 0 && limit_ns <= 10000000000LL, CODA_ERR_SHAPE);
  int dev = 0;
  DevInfo* info = nullptr;
  coda_status_t st = current_device(&dev, &info);
  if (st != CODA_OK) return st;
  bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint64_t>(limit_ns),
                                                                                gave_up_dev);
  return cudaGetLastError() == cudaSuccess ? CODA_OK : CODA_ERR_LAUNCH;
}

// ------------------------------------------------------------- FP8 (e4m3)

coda_status_t coda_fp8_quantize(const uint16_t* src, int64_t rows, int64_t cols, int transpose, uint8_t* dst,
                                float* amax_out, float* scale_out, void* stream) {
  CODA_CHECK(rows >= 0 && rows < (int64_t(1) << 31) && dim_ok(cols) && (!transpose || rows % 4 == 0) &&
                 (!transpose || rows <= int64_t(65535) * kQT),
             CODA_ERR_SHAPE);
  CODA_CHECK(src && dst && amax_out && scale_out, CODA_ERR_NULL);
  CODA_CHECK(al16(src) && al16(dst) && al16(amax_out) && al16(scale_out), CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(amax_out, 0, sizeof(float), s) != cudaSuccess) return CODA_ERR_LAUNCH;
  const size_t n8 = static_cast<size_t>(rows) * static_cast<size_t>(cols) / 8;
  if (n8 > 0) {
    const int grid = info->sms * 4;
    amax_bf16_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16*>(src), n8,
                                          reinterpret_cast<unsigned*>(amax_out));
    if (transpose) {
      const dim3 g(static_cast<unsigned>((cols + kQT - 1) / kQT), static_cast<unsigned>((rows + kQT - 1) / kQT));
      quantize_e4m3_t_kernel<<<g, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16*>(src), static_cast<int>(rows),
                                               static_cast<int>(cols), amax_out, dst);
    } else {
      quantize_e4m3_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16*>(src), n8, amax_out, dst);
    }
  }
  fp8_scale_kernel<<<1, 1, 0, s>>>(amax_out, scale_out);
  return cudaGetLastError() == cudaSuccess ? CODA_OK : CODA_ERR_LAUNCH;
}

coda_status_t coda_fp8_scale_from_amax(const float* amax, float* scale_out, void* stream) {
  CODA_CHECK(amax && scale_out, CODA_ERR_NULL);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  fp8_scale_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(amax, scale_out);
  return cudaGetLastError() == cudaSuccess ? CODA_OK : CODA_ERR_LAUNCH;
}

namespace {
inline bool fp8_dim_ok(int64_t v) { return dim_ok(v) && v % 16 == 0; }
}  // namespace

coda_status_t coda_gemm_res_partialrms_fp8(const uint8_t* x8, const float* sx, const uint8_t* Wt8, const float* sw,
                                           const uint16_t* res, const uint16_t* gamma, const float* s_hg,
                                           uint16_t* h_out, uint8_t* hg8_out, float* amax_out, float* partial,
                                           int64_t M, int64_t N, int64_t K, void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && fp8_dim_ok(N) && fp8_dim_ok(K), CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(x8 && sx && Wt8 && sw && gamma && s_hg && hg8_out && amax_out && partial, CODA_ERR_NULL);
  CODA_CHECK(al16(x8) && al16(Wt8) && al16(res) && al16(gamma) && al16(h_out) && al16(hg8_out) && al16(partial) &&
                 al16(amax_out),
             CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  using Epi = EpiLoadStore2<2>;
  GemmParams<Epi> p{};
  bool ok = tmap2d_u8(&p.tmA, x8, K, M, K, 128, kBM) && tmap2d_u8(&p.tmB, Wt8, K, N, K, 128, 128) &&
            tmap2d_u8(&p.tmBh, Wt8, K, N, K, 128, 64) && tmap2d_u8(&p.ep.tmOut2, hg8_out, N, M, N, 128, 32) &&
            tmap2d_u8_plain(&p.ep.tmOut2h, hg8_out, N, M, N, 64, 32);
  p.has_bh = 1;
  if (h_out) ok = ok && map_out_bf16(&p.ep.tmOut1, h_out, M, N, N);
  if (!ok) return CODA_ERR_INTERNAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(amax_out, 0, sizeof(float), s) != cudaSuccess) return CODA_ERR_LAUNCH;
  p.ep.in = reinterpret_cast<const __nv_bfloat16*>(res);
  p.ep.gamma = reinterpret_cast<const __nv_bfloat16*>(gamma);
  p.ep.partial = partial;
  p.ep.has_out1 = h_out != nullptr;
  p.ep.has_out2 = 1;
  p.ep.sa = sx;
  p.ep.sb = sw;
  p.ep.s_out = s_hg;
  p.ep.amax = reinterpret_cast<unsigned*>(amax_out);
  const int n_nt = static_cast<int>((N + 255) / 256);
  return run_gemm<256, pair_stages<Epi>(), false, false, true, Epi>(dev, info, p, static_cast<int>(M),
                                                                    static_cast<int>(N), static_cast<int>(K), n_nt,
                                                                    raster_group(M, N, K), kKindResPartialF8, s);
}

coda_status_t coda_gemm_rowscale_partial_fp8(const uint8_t* A8, const float* sa, const uint8_t* Wt8, const float* sw,
                                             const float* partial, int64_t T, int64_t N_norm, float eps,
                                             float* r_out, uint16_t* out, int64_t M, int64_t N, int64_t K,
                                             void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && dim_ok(N) && fp8_dim_ok(K) && T > 0 && T <= 1 << 20 &&
                 N_norm > 0 && eps >= 0.f,
             CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(A8 && sa && Wt8 && sw && partial && out, CODA_ERR_NULL);
  CODA_CHECK(al16(A8) && al16(Wt8) && al16(partial) && al16(r_out) && al16(out), CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  using Epi = EpiRowScaleF8;
  GemmParams<Epi> p{};
  if (!(tmap2d_u8(&p.tmA, A8, K, M, K, 128, kBM) && tmap2d_u8(&p.tmB, Wt8, K, N, K, 128, 128) &&
        map_out_bf16(&p.ep.tmOut, out, M, N, N)))
    return CODA_ERR_INTERNAL;
  p.ep.partial = partial;
  p.ep.T = static_cast<int>(T);
  p.ep.inv_n = 1.0f / static_cast<float>(N_norm);
  p.ep.eps = eps;
  p.ep.r_out = r_out;
  p.ep.sa = sa;
  p.ep.sb = sw;
  const int n_nt = static_cast<int>((N + 255) / 256);
  return run_gemm<256, pair_stages<Epi>(), false, false, true, Epi>(dev, info, p, static_cast<int>(M),
                                                                    static_cast<int>(N), static_cast<int>(K), n_nt,
                                                                    raster_group(M, N, K), kKindRowScaleF8,
                                                                    static_cast<cudaStream_t>(stream));
}

coda_status_t coda_gemm_fp8(const uint8_t* A8, const float* sa, const uint8_t* Wt8, const float* sw, uint16_t* out,
                            int64_t M, int64_t N, int64_t K, void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && dim_ok(N) && fp8_dim_ok(K), CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(A8 && sa && Wt8 && sw && out, CODA_ERR_NULL);
  CODA_CHECK(al16(A8) && al16(Wt8) && al16(out), CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  using Epi = EpiRowScaleF8;
  GemmParams<Epi> p{};
  if (!(tmap2d_u8(&p.tmA, A8, K, M, K, 128, kBM) && tmap2d_u8(&p.tmB, Wt8, K, N, K, 128, 128) &&
        map_out_bf16(&p.ep.tmOut, out, M, N, N)))
    return CODA_ERR_INTERNAL;
  p.ep.sa = sa;
  p.ep.sb = sw;
  const int n_nt = static_cast<int>((N + 255) / 256);
  return run_gemm<256, pair_stages<Epi>(), false, false, true, Epi>(dev, info, p, static_cast<int>(M),
                                                                    static_cast<int>(N), static_cast<int>(K), n_nt,
                                                                    raster_group(M, N, K), kKindRowScaleF8,
                                                                    static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------ block-scaled e4m3 (MXFP8)

int64_t coda_mx_sf_bytes(int64_t rows, int64_t cols, int operand) {
  if (rows < 0 || cols < 0 || cols % 128 != 0 || (operand != 0 && operand != 1)) return -1;
  const int64_t nkb = cols / 128;
  // A: a 512-byte atom per (k-block, 128-row block); B: a 4 KB image per (k-block, 256-row tile)
  return operand == 0 ? nkb * ((rows + 127) / 128) * 512 : nkb * ((rows + 255) / 256) * 4096;
}

namespace {
inline bool mx_dim_ok(int64_t v) { return dim_ok(v) && v % 128 == 0; }
}  // namespace

coda_status_t coda_mx_quantize(const uint16_t* src, int64_t rows, int64_t cols, int operand, uint8_t* q_out,
                               uint8_t* sf_out, void* stream) {
  CODA_CHECK(rows >= 0 && rows < (int64_t(1) << 30) && mx_dim_ok(cols) && (operand == 0 || operand == 1) &&
                 (rows + 255) / 256 * 256 * (cols / 32) < (int64_t(1) << 40),
             CODA_ERR_SHAPE);
  if (rows == 0) return CODA_OK;
  CODA_CHECK(src && q_out && sf_out, CODA_ERR_NULL);
  CODA_CHECK(al16(src) && al16(q_out) && al16(sf_out), CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  mx_quantize_kernel<<<info->sms * 4, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const __nv_bfloat16*>(src), static_cast<int>(rows), static_cast<int>(cols), operand, q_out,
      sf_out);
  return cudaGetLastError() == cudaSuccess ? CODA_OK : CODA_ERR_LAUNCH;
}

coda_status_t coda_gemm_res_partialrms_mx(const uint8_t* x8, const float* sx, const uint8_t* Wt8, const float* sw,
                                          const uint16_t* res, const uint16_t* gamma, uint16_t* h_out,
                                          uint8_t* hq_out, uint8_t* hsf_out, float* partial, int64_t M, int64_t N,
                                          int64_t K, void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && mx_dim_ok(N) && fp8_dim_ok(K), CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(x8 && sx && Wt8 && sw && gamma && hq_out && hsf_out && partial, CODA_ERR_NULL);
  CODA_CHECK(al16(x8) && al16(Wt8) && al16(res) && al16(gamma) && al16(h_out) && al16(hq_out) && al16(hsf_out) &&
                 al16(partial),
             CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  using Epi = EpiLoadStore2<3>;
  GemmParams<Epi> p{};
  bool ok = tmap2d_u8(&p.tmA, x8, K, M, K, 128, kBM) && tmap2d_u8(&p.tmB, Wt8, K, N, K, 128, 128) &&
            tmap2d_u8(&p.tmBh, Wt8, K, N, K, 128, 64) && tmap2d_u8(&p.ep.tmOut2, hq_out, N, M, N, 128, 32) &&
            tmap2d_u8_plain(&p.ep.tmOut2h, hq_out, N, M, N, 64, 32);
  p.has_bh = 1;
  if (h_out) ok = ok && map_out_bf16(&p.ep.tmOut1, h_out, M, N, N);
  if (!ok) return CODA_ERR_INTERNAL;
  p.ep.in = reinterpret_cast<const __nv_bfloat16*>(res);
  p.ep.gamma = reinterpret_cast<const __nv_bfloat16*>(gamma);
  p.ep.partial = partial;
  p.ep.has_out1 = h_out != nullptr;
  p.ep.has_out2 = 1;
  p.ep.sa = sx;
  p.ep.sb = sw;
  p.ep.sf_out = hsf_out;
  p.ep.sf_rb = static_cast<int>((M + 127) / 128);
  const int n_nt = static_cast<int>((N + 255) / 256);
  return run_gemm<256, pair_stages<Epi>(), false, false, true, Epi>(dev, info, p, static_cast<int>(M),
                                                                    static_cast<int>(N), static_cast<int>(K), n_nt,
                                                                    raster_group(M, N, K), kKindResPartialMX,
                                                                    static_cast<cudaStream_t>(stream));
}

coda_status_t coda_gemm_rowscale_partial_mx(const uint8_t* Aq, const uint8_t* Asf, const uint8_t* Wq,
                                            const uint8_t* Wsf, const float* partial, int64_t T, int64_t N_norm,
                                            float eps, float* r_out, uint16_t* out, int64_t M, int64_t N, int64_t K,
                                            void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && mx_dim_ok(N) && mx_dim_ok(K) &&
                 (partial == nullptr || (T > 0 && T <= 1 << 20 && N_norm > 0 && eps >= 0.f)),
             CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(Aq && Asf && Wq && Wsf && out, CODA_ERR_NULL);
  CODA_CHECK(al16(Aq) && al16(Asf) && al16(Wq) && al16(Wsf) && al16(partial) && al16(r_out) && al16(out),
             CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  using Epi = EpiRowScaleMX;
  GemmParams<Epi> p{};
  // scales as rows of 512 bytes: A's atoms (one row each), B's 4 KB images (8 rows)
  const int64_t rba = (M + 127) / 128, ntl = (N + 255) / 256, nkb = K / 128;
  if (!(tmap2d_u8(&p.tmA, Aq, K, M, K, 128, kBM) && tmap2d_u8(&p.tmB, Wq, K, N, K, 128, 128) &&
        tmap_sf(&p.tmSFA, Asf, static_cast<uint64_t>(nkb * rba), 1) &&
        tmap_sf(&p.tmSFB, Wsf, static_cast<uint64_t>(nkb * ntl * 8), 8) && map_out_bf16(&p.ep.tmOut, out, M, N, N)))
    return CODA_ERR_INTERNAL;
  p.sf_rba = static_cast<int>(rba);
  p.sf_ntl = static_cast<int>(ntl);
  p.ep.partial = partial;
  p.ep.T = static_cast<int>(T);
  p.ep.inv_n = partial ? 1.0f / static_cast<float>(N_norm) : 1.0f;
  p.ep.eps = eps;
  p.ep.r_out = partial ? r_out : nullptr;
  const int n_nt = static_cast<int>((N + 255) / 256);
  return run_gemm<256, pair_stages<Epi>(), false, false, true, Epi>(dev, info, p, static_cast<int>(M),
                                                                    static_cast<int>(N), static_cast<int>(K), n_nt,
                                                                    raster_group(M, N, K), kKindRowScaleMX,
                                                                    static_cast<cudaStream_t>(stream));
}

coda_status_t coda_unfused_rmsnorm_fp8(const uint16_t* h, const uint16_t* gamma, float eps, const float* s_y,
                                       uint8_t* y8_out, float* amax_out, float* r_out, int64_t M, int64_t N,
                                       void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && fp8_dim_ok(N) && eps >= 0.f, CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(h && gamma && s_y && y8_out && amax_out, CODA_ERR_NULL);
  CODA_CHECK(al16(h) && al16(gamma) && al16(y8_out) && al16(amax_out) && al16(r_out), CODA_ERR_ALIGN);
  int dev = 0;
  DevInfo* info = nullptr;
  coda_status_t st = current_device(&dev, &info);
  if (st != CODA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(amax_out, 0, sizeof(float), s) != cudaSuccess) return CODA_ERR_LAUNCH;
  rmsnorm_e4m3_kernel<<<static_cast<int>(M), kNormThreads, 0, s>>>(
      reinterpret_cast<const __nv_bfloat16*>(h), reinterpret_cast<const __nv_bfloat16*>(gamma), eps, s_y, y8_out,
      r_out, reinterpret_cast<unsigned*>(amax_out), static_cast<int>(N));
  return cudaGetLastError() == cudaSuccess ? CODA_OK : CODA_ERR_LAUNCH;
}

// ------------------------------------------------- host-buffer block pipeline

}  // extern "C"

namespace {

// Streams and events of the host-buffer pipeline, created once per device.
// `mu` is held while a call enqueues its work: the events are re-recorded by
// every call, and a wait must see the record of its own call, not one made
// at the same time by another host thread on another stream.
struct HostPipe {
  std::mutex mu;
  bool init = false;
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t start = nullptr;
  cudaEvent_t in_done[2] = {}, comp_done[2] = {}, out_done[2] = {};
};
HostPipe g_pipe[64];

coda_status_t host_pipe(int dev, HostPipe** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  HostPipe& hp = g_pipe[dev];
  if (!hp.init) {
    bool ok = cudaStreamCreateWithFlags(&hp.s_in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.s_out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < 2; ++i)
      ok = cudaEventCreateWithFlags(&hp.in_done[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&hp.comp_done[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&hp.out_done[i], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
      cudaGetLastError();
      return CODA_ERR_LAUNCH;
    }
    hp.init = true;
  }
  *out = &hp;
  return CODA_OK;
}

// Per-slot buffers of one chunk of chunk_rows rows.
struct HostSlot {
  uint16_t *x, *res, *h, *hg, *out;
  float *partial, *r;
};

size_t host_slot_bytes(int64_t C, int64_t K, int64_t N, int64_t N2) {
  const size_t T = static_cast<size_t>(coda_partial_cols(N));
  return align256(static_cast<size_t>(C * K) * 2) + 3 * align256(static_cast<size_t>(C * N) * 2) +
         align256(static_cast<size_t>(C * N2) * 2) + align256(T * static_cast<size_t>(C) * 4) +
         align256(static_cast<size_t>(C) * 4);
}

HostSlot host_slot(void* base, int64_t C, int64_t K, int64_t N, int64_t N2) {
  const size_t T = static_cast<size_t>(coda_partial_cols(N));
  uint8_t* p = static_cast<uint8_t*>(base);
  HostSlot sl;
  sl.x = reinterpret_cast<uint16_t*>(p);
  p += align256(static_cast<size_t>(C * K) * 2);
  sl.res = reinterpret_cast<uint16_t*>(p);
  p += align256(static_cast<size_t>(C * N) * 2);
  sl.h = reinterpret_cast<uint16_t*>(p);
  p += align256(static_cast<size_t>(C * N) * 2);
  sl.hg = reinterpret_cast<uint16_t*>(p);
  p += align256(static_cast<size_t>(C * N) * 2);
  sl.out = reinterpret_cast<uint16_t*>(p);
  p += align256(static_cast<size_t>(C * N2) * 2);
  sl.partial = reinterpret_cast<float*>(p);
  p += align256(T * static_cast<size_t>(C) * 4);
  sl.r = reinterpret_cast<float*>(p);
  return sl;
}

}  // namespace

extern "C" {

size_t coda_rmsnorm_block_host_workspace_size(int64_t K, int64_t N, int64_t N2, int64_t chunk_rows) {
  if (chunk_rows <= 0 || K <= 0 || N <= 0 || N2 <= 0) return 0;
  return 2 * host_slot_bytes(chunk_rows, K, N, N2);
}

coda_status_t coda_rmsnorm_block_host(const uint16_t* x_host, const uint16_t* res_host, const uint16_t* W1,
                                      const uint16_t* W2, const uint16_t* gamma, float eps, uint16_t* out_host,
                                      void* ws, size_t ws_bytes, int64_t M, int64_t K, int64_t N, int64_t N2,
                                      int64_t chunk_rows, void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && dim_ok(K) && dim_ok(N) && dim_ok(N2) && eps >= 0.f &&
                 chunk_rows > 0 && chunk_rows % 256 == 0,
             CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(x_host && W1 && W2 && gamma && out_host && ws, CODA_ERR_NULL);
  CODA_CHECK(al16(W1) && al16(W2) && al16(gamma) && al16(ws), CODA_ERR_ALIGN);
  CODA_CHECK(ws_bytes >= coda_rmsnorm_block_host_workspace_size(K, N, N2, chunk_rows), CODA_ERR_WORKSPACE);
  int dev = 0;
  DevInfo* info = nullptr;
  {
    const coda_status_t ds = current_device(&dev, &info);
    if (ds != CODA_OK) return ds;
  }
  HostPipe* hp = nullptr;
  {
    const coda_status_t ps = host_pipe(dev, &hp);
    if (ps != CODA_OK) return ps;
  }
  std::lock_guard<std::mutex> call_lock(hp->mu);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t slot_bytes = host_slot_bytes(chunk_rows, K, N, N2);
  const HostSlot slot[2] = {host_slot(ws, chunk_rows, K, N, N2),
                            host_slot(static_cast<uint8_t*>(ws) + slot_bytes, chunk_rows, K, N, N2)};
  // nothing of this call runs before the caller's earlier work on `stream`
  bool ok = cudaEventRecord(hp->start, s) == cudaSuccess && cudaStreamWaitEvent(hp->s_in, hp->start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(hp->s_out, hp->start, 0) == cudaSuccess;
  const int64_t nchunks = (M + chunk_rows - 1) / chunk_rows;
  coda_status_t st = CODA_OK;
  // On an error part-way: the copies already queued on the library's streams
  // still end before anything the caller queues on `stream` after this call.
  auto drain = [&]() {
    if (cudaEventRecord(hp->in_done[0], hp->s_in) == cudaSuccess) cudaStreamWaitEvent(s, hp->in_done[0], 0);
    if (cudaEventRecord(hp->out_done[0], hp->s_out) == cudaSuccess) cudaStreamWaitEvent(s, hp->out_done[0], 0);
  };
  for (int64_t i = 0; ok && i < nchunks; ++i) {
    const int b = static_cast<int>(i & 1);
    const HostSlot& sl = slot[b];
    const int64_t r0 = i * chunk_rows;
    const int64_t rows = M - r0 < chunk_rows ? M - r0 : chunk_rows;
    // inputs of chunk i into slot b, once chunk i - 2 has finished computing from it
    if (i >= 2) ok = ok && cudaStreamWaitEvent(hp->s_in, hp->comp_done[b], 0) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(sl.x, x_host + r0 * K, static_cast<size_t>(rows * K) * 2, cudaMemcpyHostToDevice,
                               hp->s_in) == cudaSuccess;
    if (res_host)
      ok = ok && cudaMemcpyAsync(sl.res, res_host + r0 * N, static_cast<size_t>(rows * N) * 2,
                                 cudaMemcpyHostToDevice, hp->s_in) == cudaSuccess;
    ok = ok && cudaEventRecord(hp->in_done[b], hp->s_in) == cudaSuccess;
    // the block on the caller's stream, once the inputs are in and the output
    // slot has been copied out (chunk i - 2)
    ok = ok && cudaStreamWaitEvent(s, hp->in_done[b], 0) == cudaSuccess;
    if (i >= 2) ok = ok && cudaStreamWaitEvent(s, hp->out_done[b], 0) == cudaSuccess;
    if (!ok) break;
    st = coda_gemm_res_partialrms(sl.x, W1, res_host ? sl.res : nullptr, gamma, sl.h, sl.hg, sl.partial, rows, N, K,
                                  s);
    if (st == CODA_OK)
      st = coda_gemm_rowscale_partial(sl.hg, W2, sl.partial, coda_partial_cols(N), N, eps, sl.r, sl.out, rows, N2, N, s);
    if (st != CODA_OK) {
      drain();
      return st;
    }
    ok = cudaEventRecord(hp->comp_done[b], s) == cudaSuccess &&
         cudaStreamWaitEvent(hp->s_out, hp->comp_done[b], 0) == cudaSuccess &&
         cudaMemcpyAsync(out_host + r0 * N2, sl.out, static_cast<size_t>(rows * N2) * 2, cudaMemcpyDeviceToHost,
                         hp->s_out) == cudaSuccess &&
         cudaEventRecord(hp->out_done[b], hp->s_out) == cudaSuccess;
  }
  // the caller's stream waits for the last copies out (and so for everything)
  ok = ok && cudaStreamWaitEvent(s, hp->out_done[(nchunks - 1) & 1], 0) == cudaSuccess;
  if (nchunks >= 2) ok = ok && cudaStreamWaitEvent(s, hp->out_done[nchunks & 1], 0) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    drain();
    return CODA_ERR_LAUNCH;
  }
  return CODA_OK;
}

}  // extern "C"

// =========================================================================
// RMSNorm backward with library-owned scratch (no allocation by anyone)
// =========================================================================
//
// coda_rms_reduce_bwd needs a scratch buffer for its per-row-block dgamma
// partials, which the caller normally allocates and passes in.  Some callers
// cannot allocate device memory when they call: for example a serving or
// training process that fixes its device-memory budget at start-up and may not
// allocate afterwards, or a host framework that owns all device memory through
// its own pool and has no way to hand out a workspace.  For them this variant
// keeps the scratch in a fixed array inside the library's device image.
//
// The array below is one static device array of kNoAllocScratchFloats floats
// (4 MiB), present on every GPU that loads this library until the process
// exits.  It is shared by every call on a device and keeps whatever the last
// call wrote; the kernels write every entry they later read, so nothing in it
// has to start at zero.  Two calls whose kernels run at the same time on one
// device (different streams, or different host threads) race on the array and
// must be ordered by the caller.

namespace {

constexpr size_t kNoAllocScratchFloats = size_t(1) << 20;

float* g_noalloc_scratch[64] = {};  // per-device device address of the array

}  // namespace

static __device__ __align__(256) float g_coda_rms_bwd_scratch[kNoAllocScratchFloats];

namespace {

// Device address of the scratch array on device `dev` (which must be current).
// The first call on a device looks it up; host code cannot use the array's
// name as a device pointer.
coda_status_t noalloc_scratch_on(int dev, float** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_noalloc_scratch[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_coda_rms_bwd_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return CODA_ERR_LAUNCH;
    }
    g_noalloc_scratch[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_scratch[dev];
  return CODA_OK;
}

}  // namespace

extern "C" coda_status_t coda_rms_reduce_bwd_noalloc(const float* pdr, const float* r, const float* d_hg,
                                                     const uint16_t* h, const uint16_t* gamma, uint16_t* dh_out,
                                                     float* dgamma_out, int64_t M, int64_t T, int64_t N,
                                                     void* stream) {
  CODA_CHECK(M >= 0 && M < (int64_t(1) << 31) && T > 0 && T <= 1 << 20 && dim_ok(N), CODA_ERR_SHAPE);
  if (M == 0) return CODA_OK;
  CODA_CHECK(pdr && r && d_hg && h && gamma && dh_out && dgamma_out, CODA_ERR_NULL);
  CODA_CHECK(al16(pdr) && al16(r) && al16(d_hg) && al16(h) && al16(gamma) && al16(dh_out) && al16(dgamma_out),
             CODA_ERR_ALIGN);
  const int64_t nblk = (M + kBwdRows - 1) / kBwdRows;
  CODA_CHECK(static_cast<uint64_t>(nblk) * static_cast<uint64_t>(N) <= kNoAllocScratchFloats, CODA_ERR_WORKSPACE);
  int dev = 0;
  DevInfo* info = nullptr;
  coda_status_t st = current_device(&dev, &info);
  if (st != CODA_OK) return st;
  float* part = nullptr;
  st = noalloc_scratch_on(dev, &part);
  if (st != CODA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  rms_reduce_bwd_kernel<<<static_cast<int>(nblk), kBwdThreads, 0, s>>>(
      pdr, r, d_hg, reinterpret_cast<const __nv_bfloat16*>(h), reinterpret_cast<const __nv_bfloat16*>(gamma),
      reinterpret_cast<__nv_bfloat16*>(dh_out), part, static_cast<int>(M), static_cast<int>(T), static_cast<int>(N));
  if (cudaGetLastError() != cudaSuccess) return CODA_ERR_LAUNCH;
  dgamma_final_kernel<<<static_cast<int>((N + kDgCols - 1) / kDgCols), kDgCols * kDgGroups, 0, s>>>(part, static_cast<int>(nblk),
                                                                        static_cast<int>(N), dgamma_out);
  return cudaGetLastError() == cudaSuccess ? CODA_OK : CODA_ERR_LAUNCH;
}
