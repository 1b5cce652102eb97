// Persistent, warp-specialised tcgen05 GEMM with programmable epilogues.
//
// This is the "fixed mainloop + programmable epilogue" structure of the KuCoin
// news flash "CODA: new research optimizes transformer training with GEMM
// epilogue programming" (section "CODA: the secret in the epilogue": a GEMM is
// a mainloop of tiled multiply-accumulate and an epilogue that post-processes
// the tile while it is still on chip; section "Five kinds of building blocks":
// the mainloop stays fixed and the epilogue is composed of elementwise
// transforms, vector loads, matrix-block loads/stores, chunk reductions and
// stateful transforms).
//
// Mainloop (one CTA per SM, 192 threads):
//   warp 0  - one thread issues TMA loads of A and B k-blocks into a ring of
//             shared-memory stages (128-byte swizzle).
//   warp 1  - one thread issues tcgen05.mma (bf16 x bf16 -> fp32) into one of
//             two tensor-memory accumulators (128 lanes x BN columns each).
//   warps 2-5 - the epilogue: each warp owns 32 accumulator rows (the TMEM
//             lane quarter warp % 4), reads its rows with tcgen05.ld while the
//             MMA warp already fills the other accumulator, and runs the
//             epilogue functor.  One thread owns one output row, so per-row
//             reductions (partial sums of squares, online max / sum-exp) are
//             thread-local.
// Tiles are handed out round-robin over a grouped raster (group_m M-tiles per
// column sweep) so that concurrently running CTAs share operand tiles in L2.
// Operands: A is [M, K] K-major (row-major activations) or MN-major (a
// transposed view for weight gradients); B is [K, N] MN-major (row-major
// weights) or K-major (a transposed weight).  Rows beyond M, columns beyond N
// and k beyond K are zero-filled by TMA and clipped on store.
#pragma once

#include "coda_device.cuh"
#include "coda_rowops.cuh"

namespace coda {

constexpr int kBM = 128;        // accumulator rows per tile (TMEM lanes)
constexpr int kBK = 64;         // k-block: 64 bf16 = one 128-byte swizzle row
constexpr int kThreads = 192;   // 6 warps
constexpr int kEpiWarps = 4;

struct TileSched {
  int n_mt;     // M tiles
  int n_nt;     // N tiles
  int group_m;  // M tiles per raster group
  int ntiles;
  // The last `nsplit` tiles in raster order are handed out as two units each,
  // so that a last partial wave of whole tiles on under half of the CTA pairs
  // becomes a wave of half units on all of them (0: every unit is a whole
  // tile).  kmode 0: the halves are the tile's two 128-column halves; kmode
  // 1: they are full-width tiles over the first and the second half of the
  // k-blocks, whose epilogues add their results into a zeroed output.
  int nsplit;
  int kmode;

  __device__ __forceinline__ int nunits() const { return ntiles + nsplit; }

  // Unit u -> tile (mb, nb) and half (-1 for a whole tile, else 0 or 1).
  __host__ __device__ __forceinline__ void map_unit(int u, int& mb, int& nb, int& half) const {
    const int s0 = ntiles - nsplit;
    int t = u;
    half = -1;
    if (u >= s0) {
      t = s0 + ((u - s0) >> 1);
      half = (u - s0) & 1;
    }
    map(t, mb, nb);
  }

  __host__ __device__ __forceinline__ void map(int t, int& mb, int& nb) const {
    const int per_group = group_m * n_nt;
    const int g = t / per_group;
    const int first = g * group_m;
    const int gs = n_mt - first < group_m ? n_mt - first : group_m;
    const int r = t - g * per_group;
    mb = first + r % gs;
    nb = r / gs;
  }
};

// Operand type of the mainloop: bf16 (kind::f16) unless the epilogue declares
// kFp8 = true (e4m3 operands, kind::f8f6f4).  A k-block is 128 bytes of K per
// row either way: 64 bf16 or 128 e4m3 elements.
template <class E, class = void>
struct epi_fp8 {
  static constexpr bool value = false;
};
template <class E>
struct epi_fp8<E, decltype(void(E::kFp8))> {
  static constexpr bool value = E::kFp8;
};

// Epilogue warps: 4 (one per TMEM lane quarter) unless the epilogue declares
// kWarps = 8 (two per lane quarter, each taking half of the tile's columns,
// for epilogues whose work outlasts the mainloop of a tile).
template <class E, class = void>
struct epi_warps {
  static constexpr int value = kEpiWarps;
};
template <class E>
struct epi_warps<E, decltype(void(E::kWarps))> {
  static constexpr int value = E::kWarps;
};

// Epilogues that declare kSplitN = true take a column range of 128 (a half
// tile, c.cbeg = 0 or 128) as well as whole tiles; the host may then split
// the last partial wave (TileSched::nsplit).
template <class E, class = void>
struct epi_split {
  static constexpr bool value = false;
};
template <class E>
struct epi_split<E, decltype(void(E::kSplitN))> {
  static constexpr bool value = E::kSplitN;
};

// Epilogues that declare kSplitK = true produce outputs linear in the
// accumulator, in fp32 (c.khalf >= 0: they add into the output, which the
// host has zeroed), so the split last wave may divide a tile's k-blocks
// instead of its columns (TileSched::kmode).
template <class E, class = void>
struct epi_ksplit {
  static constexpr bool value = false;
};
template <class E>
struct epi_ksplit<E, decltype(void(E::kSplitK))> {
  static constexpr bool value = E::kSplitK;
};

// Epilogues that declare kMX = true take block-scaled e4m3 operands
// (MXFP8: kind::mxf8f6f4.block_scale, an E8M0 scale per 32 elements of K,
// loaded with every k-block -- A's as a 512-byte atom, B's as a 4 KB copy
// image -- and copied into tensor memory beside the accumulator).  The
// scales take tensor-memory columns, so the tile keeps one 256-column
// accumulator instead of two; the epilogue frees it as soon as it has read
// it (arriving on TileCtx::trel itself) and writes the tile out while the
// next tile's MMAs run.
template <class E, class = void>
struct epi_mx {
  static constexpr bool value = false;
};
template <class E>
struct epi_mx<E, decltype(void(E::kMX))> {
  static constexpr bool value = E::kMX;
};

// Epilogues that declare kHasPre = true give their warps work to do before
// the first tile (Epi::pre), while that tile's mainloop runs.
template <class E, class = void>
struct epi_pre {
  static constexpr bool value = false;
};
template <class E>
struct epi_pre<E, decltype(void(E::kHasPre))> {
  static constexpr bool value = E::kHasPre;
};

template <class Epi>
struct GemmParams {
  CUtensorMap tmA;
  CUtensorMap tmB;
  CUtensorMap tmB2;  // second half of a paired B operand (SwiGLU up columns)
  CUtensorMap tmBh;  // K-major B with a 64-row box: this CTA's columns of a half tile
  int has_bh;        // tmBh is encoded (a K-major B may then be split into half tiles)
  typename Epi::Params ep;
  int M, N, K;       // GEMM sizes; N counts accumulator columns of the output space
  TileSched sched;
  uint64_t wait_ns;
  // Programmatic dependent launch (set for every CTA-pair launch):
  // pdl_trigger lets the next kernel on the stream, if launched with
  // programmatic serialisation, start its prologue on SMs this grid has left;
  // pdl_wait makes this grid wait, after its own prologue and before any
  // global read, until the previous grid has completed and its writes are
  // visible (a hardware dependency, like stream order).
  int pdl_trigger, pdl_wait;
  // Block-scaled operands: the scales of A and B seen as rows of 128 words
  // (512 bytes): A's atom kb * sf_rba + this CTA's row block (one row), B's
  // image kb * sf_ntl + the tile's column block (4 KB = 8 rows).
  CUtensorMap tmSFA;
  CUtensorMap tmSFB;
  int sf_rba, sf_ntl;  // 128-row blocks of A; 256-row tiles of B
};

// Per-warp context handed to the epilogue for one tile.
struct TileCtx {
  int M, N;          // output rows / columns
  int mb, nb;        // tile coordinates
  int row0;          // first global row of this warp's 32 rows
  uint32_t taddr;    // TMEM address of (this warp's lane 0, accumulator column 0)
  int lane;
  uint8_t* wsmem;    // this warp's epilogue shared memory
  uint64_t* wbars;   // this warp's epilogue mbarriers
  bool has_next;     // this CTA has another tile after this one
  int nrow0, ncol0;  // first row of this warp / first column of that next tile
  // Column range of the tile this warp handles, in accumulator columns: all
  // of it; with eight epilogue warps one half (`split`, `half`); or, for a
  // half-tile unit of the split last wave, the 128 columns it computed.
  int cbeg = 0, cend = 256;
  int khalf = -1;  // a K-half unit (0 or 1, TileSched::kmode): add the result into the output
  bool split = false;
  int half = 0;
  // With eight warps, a half-tile unit gives each warp 64 of a partial slot's
  // 128 columns: the second warp of a lane quarter hands its row sums to the
  // first through `xchg` (32 floats) behind the single-use mbarrier `xbar`
  // (a CTA pair runs at most one half-tile unit).  Null otherwise.
  float* xchg = nullptr;
  uint64_t* xbar = nullptr;
  // Block-scaled tiles: the cluster address of the accumulator-empty barrier
  // (on rank 0), on which the epilogue releases the accumulator itself.
  uint32_t trel = 0;
};

template <int BN, int STAGES, bool PAIR, class Epi>
struct GemmSmem {
  static constexpr int kEW = epi_warps<Epi>::value;
  static constexpr int kABytes = kBM * kBK * 2;                     // this CTA's 128 rows of A
  static constexpr int kBBytes = (PAIR ? BN / 2 : BN) * kBK * 2;    // this CTA's columns of B
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kEpiBytes = kEW * Epi::kSmemPerWarp;
  static constexpr bool kHalfXchg = kEW == 8 && epi_split<Epi>::value;  // see TileCtx::xchg
  static constexpr int kXchgBytes = kHalfXchg ? 4 * 32 * 4 : 0;
  // block-scaled operands: per stage this CTA's A-scale atom and the tile's B-scale image
  static constexpr int kSFStage = epi_mx<Epi>::value ? 512 + 4096 : 0;
  static constexpr int kNumBars = 2 * STAGES + 2 + 2 + 1 + kEW * Epi::kBarsPerWarp + (kHalfXchg ? 4 : 0);
  static constexpr int kBytes = 1024 /*align slack*/ + STAGES * kStageBytes + kEpiBytes + STAGES * kSFStage +
                                kXchgBytes + kNumBars * 8 + 16;
  static_assert(kEW == 4 || kEW == 8, "four or eight epilogue warps");
  static_assert(Epi::kSmemPerWarp % 1024 == 0, "per-warp epilogue buffers keep the 128-byte swizzle alignment");
};

// Bounded wait that ignores the abort flag (used to drain copies in flight
// before the CTA exits).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  int dummy_abort = 0;
  WaitCtx w{&dummy_abort, limit_ns};
  (void)mbar_wait(bar, parity, w);
}

// PAIR = false: one CTA per 128 x BN tile (tcgen05 cta_group::1).
// PAIR = true: a cluster of two CTAs per 256 x BN tile (cta_group::2); CTA
// rank r owns accumulator rows [128 r, 128 r + 128) of the tile and loads its
// own 128 rows of A and its own BN/2 columns of B.  Rank 0 issues the MMAs,
// waits for both CTAs' copies on its full barriers (the copies of rank 1
// complete there), and its commits arrive on the barriers of both CTAs.
template <int BN, int STAGES, bool A_MN, bool B_MN, bool PAIR, class Epi>
__global__ void __launch_bounds__(64 + 32 * epi_warps<Epi>::value, 1)
    coda_gemm_kernel(const __grid_constant__ GemmParams<Epi> p) {
  using S = GemmSmem<BN, STAGES, PAIR, Epi>;
  constexpr int kEW = S::kEW;
  static_assert(BN % 64 == 0 && BN <= 256, "BN must be a multiple of 64, at most 256");
  static_assert(2 * BN == 512 || 2 * BN == 256 || 2 * BN == 128, "TMEM columns must be a power of two");
  static_assert(!PAIR || BN == 256, "pair tiles are 256 x 256");
  constexpr int kTileM = PAIR ? 2 * kBM : kBM;   // rows per tile
  constexpr int kBCols = PAIR ? BN / 2 : BN;     // B columns loaded by this CTA
  constexpr bool kF8 = epi_fp8<Epi>::value;
  constexpr int kKb = kF8 ? 2 * kBK : kBK;       // K elements per k-block (128 bytes per row)
  static_assert(!kF8 || (!A_MN && !B_MN && PAIR), "e4m3 operands: K-major A and B, CTA pairs");
  constexpr bool kSplit = epi_split<Epi>::value;
  static_assert(!kSplit || (PAIR && !Epi::kPairedB), "half tiles: CTA pairs, unpaired B");
  constexpr bool kMX = epi_mx<Epi>::value;
  static_assert(!kMX || (kF8 && !kSplit && !epi_ksplit<Epi>::value && BN == 256),
                "block-scaled tiles: e4m3 CTA pairs, whole 256-column tiles");
  constexpr int kAccBufs = kMX ? 1 : 2;  // accumulators in tensor memory
  constexpr uint32_t kSFCol = 256;       // block-scaled: first scale column (after the accumulator)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * S::kABytes;
  uint8_t* sEpi = smem + STAGES * S::kStageBytes;
  uint8_t* sSF = sEpi + S::kEpiBytes;  // block-scaled: the scale atoms of each stage
  float* sXchg = reinterpret_cast<float*>(sSF + STAGES * S::kSFStage);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sXchg) + S::kXchgBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* ebars = drain + 1;
  uint64_t* xbars = ebars + kEW * Epi::kBarsPerWarp;  // kHalfXchg: one per lane quarter
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(xbars + (S::kHalfXchg ? 4 : 0));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const int tile_step = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  const int tile_first = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], PAIR ? 2 * kEW : kEW);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < kEW * Epi::kBarsPerWarp; ++i) mbar_init(&ebars[i], 1);
    if (S::kHalfXchg)
      for (int i = 0; i < 4; ++i) mbar_init(&xbars[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmA);
    tma_prefetch_desc(&p.tmB);
    if (Epi::kPairedB) tma_prefetch_desc(&p.tmB2);
    if (kMX) {
      tma_prefetch_desc(&p.tmSFA);
      tma_prefetch_desc(&p.tmSFB);
    }
  }
  if (warp == 1) {
    if (PAIR) {
      tmem_alloc_pair(tmem_holder, 2 * BN);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_holder, 2 * BN);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync_all();  // the peer's barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const WaitCtx w{abort_flag, p.wait_ns};
  if (p.pdl_trigger) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (p.pdl_wait) asm volatile("griddepcontrol.wait;" ::: "memory");
  const int nkb = (p.K + kKb - 1) / kKb;
  const int ntiles = p.sched.nunits();  // schedule units: whole tiles, then (with nsplit) half tiles

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      const uint32_t full0 = PAIR ? mapa_shared(smem_u32(full), 0) : 0u;  // rank 0's full[0]
      for (int t = tile_first; ok && t < ntiles; t += tile_step) {
        int mb, nb, half;
        p.sched.map_unit(t, mb, nb, half);
        // a K-half unit loads the whole tile's columns over its half of the k-blocks
        const int kb_lo = (p.sched.kmode && half > 0) ? nkb / 2 : 0;
        const int kb_hi = (p.sched.kmode && half == 0) ? nkb / 2 : nkb;
        if (p.sched.kmode) half = -1;
        const int arow = mb * kTileM + static_cast<int>(rank) * kBM;  // first A row of this CTA
        // first B column of this CTA: a half tile covers BN/2 columns, kBCols/2 per CTA
        const int bcol = half < 0 ? nb * BN + static_cast<int>(rank) * kBCols
                                  : nb * BN + half * (BN / 2) + static_cast<int>(rank) * (kBCols / 2);
        for (int kb = kb_lo; kb < kb_hi; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, w)) {
            ok = false;
            break;
          }
          uint8_t* a = sA + stage * S::kABytes;
          uint8_t* b = sB + stage * S::kBBytes;
          if (PAIR) {
            if (rank == 0)
              mbar_arrive_expect_tx(&full[stage], half < 0 ? 2 * (S::kStageBytes + S::kSFStage)
                                                           : 2 * (S::kABytes + S::kBBytes / 2));
            const uint32_t fb = full0 + stage * 8;
            if (!A_MN) {
              tma_load_2d_pair(a, &p.tmA, fb, kb * kKb, arow);
            } else {
#pragma unroll
              for (int j = 0; j < kBM / 64; ++j)
                tma_load_2d_pair(a + j * (64 * kBK * 2), &p.tmA, fb, arow + j * 64, kb * kBK);
            }
            if (kSplit && half >= 0) {
              // this CTA's 64 columns of the half tile
              if (!B_MN)
                tma_load_2d_pair(b, &p.tmBh, fb, kb * kKb, bcol);
              else
                tma_load_2d_pair(b, &p.tmB, fb, bcol, kb * kBK);
            } else if (!B_MN) {
              tma_load_2d_pair(b, &p.tmB, fb, kb * kKb, bcol);
            } else if (Epi::kPairedB) {
              // rank 0 holds the gate half, rank 1 the up half of the accumulator columns
              const CUtensorMap* m = rank == 0 ? &p.tmB : &p.tmB2;
#pragma unroll
              for (int j = 0; j < kBCols / 64; ++j)
                tma_load_2d_pair(b + j * (64 * kBK * 2), m, fb, nb * (BN / 2) + j * 64, kb * kBK);
            } else {
#pragma unroll
              for (int j = 0; j < kBCols / 64; ++j)
                tma_load_2d_pair(b + j * (64 * kBK * 2), &p.tmB, fb, bcol + j * 64, kb * kBK);
            }
            if (kMX) {
              // the scales of this k-block: this CTA's 128 rows of A, the tile's 256 columns of B
              uint8_t* sf = sSF + stage * S::kSFStage;
              tma_load_2d_pair(sf, &p.tmSFA, fb, 0, kb * p.sf_rba + mb * 2 + static_cast<int>(rank));
              tma_load_2d_pair(sf + 512, &p.tmSFB, fb, 0, (kb * p.sf_ntl + nb) * 8);
            }
          } else {
            mbar_arrive_expect_tx(&full[stage], S::kStageBytes);
            if (!A_MN) {
              tma_load_2d(a, &p.tmA, &full[stage], kb * kBK, arow);
            } else {
#pragma unroll
              for (int j = 0; j < kBM / 64; ++j)
                tma_load_2d(a + j * (64 * kBK * 2), &p.tmA, &full[stage], arow + j * 64, kb * kBK);
            }
            if (!B_MN) {
              tma_load_2d(b, &p.tmB, &full[stage], kb * kBK, bcol);
            } else {
#pragma unroll
              for (int j = 0; j < BN / 64; ++j) {
                if (Epi::kPairedB) {
                  const CUtensorMap* m = (j < BN / 128) ? &p.tmB : &p.tmB2;
                  const int col = nb * (BN / 2) + (j % (BN / 128)) * 64;
                  tma_load_2d(b + j * (64 * kBK * 2), m, &full[stage], col, kb * kBK);
                } else {
                  tma_load_2d(b + j * (64 * kBK * 2), &p.tmB, &full[stage], bcol + j * 64, kb * kBK);
                }
              }
            }
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Drain: every load issued must have landed before shared memory goes
      // away.  A single CTA sees its loads complete on its full barriers; in a
      // pair they complete on rank 0's, so both CTAs wait for the MMA's release
      // of each stage instead (it follows the completion of both halves).
      const long n = issued < STAGES ? issued : STAGES;
      for (long i = 0; i < n; ++i) {
        if (stage == 0) {
          stage = STAGES - 1;
          phase ^= 1u;
        } else {
          --stage;
        }
        drain_wait(PAIR ? &empty[stage] : &full[stage], phase, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0 && rank == 0) {
      constexpr uint32_t kIdesc = kF8 ? idesc_e4m3_f32(kTileM, BN) : idesc_bf16_f32(kTileM, BN, A_MN, B_MN);
      // a half tile: N = BN / 2
      constexpr uint32_t kIdescH = kF8 ? idesc_e4m3_f32(kTileM, BN / 2) : idesc_bf16_f32(kTileM, BN / 2, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int t = tile_first; ok && t < ntiles; t += tile_step, ++it) {
        const int acc = kAccBufs == 2 ? (it & 1) : 0;
        const uint32_t aph = kAccBufs == 2 ? ((it >> 1) & 1) : (it & 1);
        int half = -1;
        if (kSplit || epi_ksplit<Epi>::value) {
          int mb_, nb_;
          p.sched.map_unit(t, mb_, nb_, half);
        }
        // a K-half unit: the whole width over its half of the k-blocks
        const int kb_lo = (p.sched.kmode && half > 0) ? nkb / 2 : 0;
        const int kb_hi = (p.sched.kmode && half == 0) ? nkb / 2 : nkb;
        if (p.sched.kmode) half = -1;
        const uint32_t idesc = (kSplit && half >= 0) ? kIdescH : kIdesc;
        if (!mbar_wait(&tempty[acc], aph ^ 1u, w)) break;
        tc_fence_after();
        // a half tile accumulates into the accumulator columns it covers
        const uint32_t d = tmem_base + acc * BN + (half > 0 ? BN / 2 : 0);
        for (int kb = kb_lo; kb < kb_hi; ++kb) {
          if (!mbar_wait(&full[stage], phase, w)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * S::kABytes);
          const uint32_t b0 = smem_u32(sB + stage * S::kBBytes);
          // block-scaled: this stage's scales go to 16 tensor-memory columns of
          // their own (A's atom at +0, B's image at +8)
          const uint32_t tsf = tmem_base + kSFCol + static_cast<uint32_t>(stage) * 16u;
          if (kMX) {
            const uint32_t sf = smem_u32(sSF + stage * S::kSFStage);
            tc_cp_32x128_w4_pair(tsf, sdesc_plain16(sf));
            tc_cp_128x256_pair(tsf + 8, sdesc_sf_image(sf + 512));
          }
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = A_MN ? sdesc_sw128(a0 + kk * 16 * 128, 64 * kBK * 2, 1024)
                                     : sdesc_sw128(a0 + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? sdesc_sw128(b0 + kk * 16 * 128, 64 * kBK * 2, 1024)
                                     : sdesc_sw128(b0 + kk * 32, 16, 1024);
            const uint32_t accum = (kb != kb_lo || kk != 0) ? 1u : 0u;
            if (kMX)
              tc_mma_mx_pair(d, ad, bd, idesc_mx_e4m3(kTileM, BN, static_cast<uint32_t>(kk)),
                             tsf | (static_cast<uint32_t>(kk) << 30), (tsf + 8) | (static_cast<uint32_t>(kk) << 30),
                             accum);
            else if (kF8)
              tc_mma_f8_pair(d, ad, bd, idesc, accum);
            else if (PAIR)
              tc_mma_bf16_pair(d, ad, bd, idesc, accum);
            else
              tc_mma_bf16(d, ad, bd, kIdesc, accum);
          }
          if (PAIR)
            tc_commit_pair_mc(&empty[stage], 0x3);
          else
            tc_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (PAIR)
          tc_commit_pair_mc(&tfull[acc], 0x3);
        else
          tc_commit(&tfull[acc]);
      }
      // All MMAs issued by this thread have completed once this arrives.
      if (PAIR)
        tc_commit_pair(drain);
      else
        tc_commit(drain);
      drain_wait(drain, 0, p.wait_ns);
    }
  } else {
    // --------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int ew = warp - 2;
    const int half = kEW == 8 ? ew >> 2 : 0;  // warps 2-5: first half of the columns, 6-9: second
    uint8_t* wsmem = sEpi + ew * Epi::kSmemPerWarp;
    uint64_t* wbars = ebars + ew * Epi::kBarsPerWarp;
    // accumulator release goes to rank 0's barriers (where the MMA waits)
    const uint32_t tempty0 = PAIR ? mapa_shared(smem_u32(tempty), 0) : 0u;
    typename Epi::State st;
    Epi::init_state(st);
    if constexpr (epi_pre<Epi>::value)
      Epi::pre(p.ep, static_cast<long long>(blockIdx.x) * kEW + ew, static_cast<long long>(gridDim.x) * kEW, lane);
    int it = 0;
    for (int t = tile_first; t < ntiles; t += tile_step, ++it) {
      int mb, nb, half_t;
      p.sched.map_unit(t, mb, nb, half_t);
      const int acc = kAccBufs == 2 ? (it & 1) : 0;
      const uint32_t aph = kAccBufs == 2 ? ((it >> 1) & 1) : (it & 1);
      // Warp-uniform outcome: tcgen05.ld below is a warp-collective instruction.
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph, w))) break;
      tc_fence_after();
      TileCtx c;
      c.M = p.M;
      c.N = p.N;
      c.mb = mb;
      c.nb = nb;
      c.row0 = mb * kTileM + static_cast<int>(rank) * kBM + q * 32;
      c.taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN;
      c.lane = lane;
      c.wsmem = wsmem;
      c.wbars = wbars;
      c.has_next = t + tile_step < ntiles;
      c.nrow0 = 0;
      c.ncol0 = 0;
      if (c.has_next) {
        int nmb, nnb, nhalf;
        p.sched.map_unit(t + tile_step, nmb, nnb, nhalf);
        c.nrow0 = nmb * kTileM + static_cast<int>(rank) * kBM + q * 32;
        c.ncol0 = nnb * BN + (nhalf > 0 && !p.sched.kmode ? BN / 2 : 0);
      }
      if (p.sched.kmode) {
        // a K-half unit covers the whole tile and adds its result into the output
        c.khalf = half_t;
        half_t = -1;
      }
      c.split = kEW == 8;
      c.half = half;
      c.cbeg = kEW == 8 ? half * (BN / 2) : 0;
      c.cend = kEW == 8 ? (half + 1) * (BN / 2) : BN;
      if (kSplit && half_t >= 0) {
        // a half tile: its 128 columns, in the accumulator columns of the same
        // range (with eight warps, 64 of them per warp)
        c.cbeg = half_t * (BN / 2) + (kEW == 8 ? half * (BN / 4) : 0);
        c.cend = c.cbeg + (kEW == 8 ? BN / 4 : BN / 2);
        if (S::kHalfXchg) {
          c.xchg = sXchg + q * 32;
          c.xbar = &xbars[q];
        }
      }
      c.trel = tempty0 + acc * 8;
      const bool ok = Epi::template tile<BN>(p.ep, c, st, w);
      if (!kMX) {  // a block-scaled epilogue has released the accumulator itself
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (PAIR)
            mbar_arrive_cluster(tempty0 + acc * 8);
          else
            mbar_arrive(&tempty[acc]);
        }
      }
      if (!ok) break;
    }
    Epi::finish(p.ep, st, wbars, lane, p.wait_ns);
  }

  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync_all();  // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    tc_fence_after();
    if (PAIR)
      tmem_dealloc_pair(tmem_base, 2 * BN);
    else
      tmem_dealloc(tmem_base, 2 * BN);
  }
}

// =========================================================================
// Epilogues
// =========================================================================

// Loads 64 accumulator columns [col, col + 64) of this thread's row.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&v0)[32], uint32_t (&v1)[32]) {
  tmem_ld32(taddr, v0);
  tmem_ld32(taddr + 32, v1);
  tmem_ld_wait(v0);
  reg_pin(v1);
}

__device__ __forceinline__ float acc_at(const uint32_t (&v0)[32], const uint32_t (&v1)[32], int i) {
  return __uint_as_float(i < 32 ? v0[i] : v1[i - 32]);
}

// ---------------------------------------------------------------------------
// Read one bf16 tile, store two tiles and a per-row partial sum.
//   MODE 0 (first GEMM of the block, "GEMM-Residual-PartialRMS"):
//     h = acc + res;  out1 = bf16(h);  out2 = hg = bf16(gamma * h);  partial += h^2
//   MODE 1 (backward of the row-scaled second GEMM, acc = P = dOut W2^T):
//     in = hg;  out1 = y = bf16(r * hg);  out2 = d_hg = r * P (fp32);  partial += hg * P
//   MODE 2 (first GEMM of the FP8 block, e4m3 operands with per-tensor scales):
//     h = acc * sa * sb + res;  out1 = bf16(h);  partial += h^2;
//     out2 = hg8 = e4m3(gamma * h / s_out) (round to nearest even, saturating);
//     amax = max |gamma * h| (the next call's scale, by atomic max on its bits)
//   MODE 3 (first GEMM of the MXFP8 block, e4m3 operands with per-tensor scales):
//     h and partial as MODE 2; out2 = hg in MXFP8: each 32-column block of
//     gamma * h gets the smallest power-of-two scale 2^e that keeps it within
//     the e4m3 range, its codes are e4m3(gamma * h * 2^-e) and the byte e + 127
//     goes to the A scale layout (sf_out) -- the scales of the data being
//     written, in the epilogue, with no scale carried over between calls
// The input tile is read straight into registers (each thread its own row)
// 32 columns ahead, and the first columns of the next tile are requested
// before this tile's last ones are processed, so their latency hides behind
// the epilogue math.  Outputs are staged in shared
// memory (128-byte swizzle) and written by TMA stores from one staging buffer
// per warp (a second buffer would cost the mainloop its sixth pipeline stage,
// which is worth more: 63.5 against 65.5 us on the 1B block's first GEMM).
// partial is laid out [128-column slot][row] (fp32).
// ---------------------------------------------------------------------------
template <int MODE>
struct EpiLoadStore2 {
  static constexpr int kNBuf = 1;
  static constexpr bool kFp8 = MODE >= 2;
  // out2 staging: 32 x 64 bf16; 32 x 64 fp32 as two 32 x 32 boxes; or 32 x 128 e4m3 (two chunks)
  static constexpr int kOut2Bytes = MODE == 1 ? 8192 : 4096;
  static constexpr int kBufBytes = 4096 + kOut2Bytes;
  static constexpr int kSmemPerWarp = kNBuf * kBufBytes;
  // Behind the e4m3 mainloop (twice the bf16 rate) the FP8 epilogue outlasts
  // a tile's MMAs: eight warps, two per lane quarter, each taking half of the
  // tile's columns (54 against 67 us on the 1B block's first GEMM).  The bf16
  // modes keep four warps and with them a sixth pipeline stage (63.5 against
  // 66.6 us with eight warps and five stages).
  static constexpr int kWarps = MODE >= 2 ? 8 : 4;
  static constexpr int kBarsPerWarp = 0;
  static constexpr bool kPairedB = false;
  // Every mode takes half tiles (the split last wave).  In the e4m3 mode a
  // half tile gives each of its eight warps 64 columns, whose codes are
  // staged as plain 64-byte rows and stored through tmOut2h.
  static constexpr bool kSplitN = true;
  // MODE 1 (the P GEMM, K = the long output width) may split its last wave
  // by k-blocks: d_hg = r P and pdr = sum hg P are linear in P, so each half
  // adds into them (zeroed by the host); y = r hg does not depend on P and
  // is stored by the first half.
  static constexpr bool kSplitK = MODE == 1;

  struct Params {
    CUtensorMap tmOut1;          // [M, N] bf16, box 64 x 32
    CUtensorMap tmOut2;          // [M, N] bf16 box 64 x 32 (MODE 0) or fp32 box 32 x 32 (MODE 1)
    CUtensorMap tmOut2h;         // MODE 2: [M, N] e4m3, box 64 x 32, no swizzle (a warp's 64 columns of a half tile)
    const __nv_bfloat16* in;     // [M, N]: res (MODE 0, may be null) or hg (MODE 1)
    const __nv_bfloat16* gamma;  // MODE 0 (may be null when out2 is not stored)
    const float* r;              // MODE 1
    float* partial;              // [T, M] or null
    int has_out1, has_out2;
    const float* sa;             // MODE 2: scales of the e4m3 operands A and B
    const float* sb;
    const float* s_out;          // MODE 2: scale hg8 is quantised with
    unsigned* amax;              // MODE 2: running max |hg| (fp32 bits; zeroed by the caller)
    uint8_t* sf_out;             // MODE 3: hg's scale bytes, A layout (N % 128 == 0)
    int sf_rb;                   // MODE 3: 128-row blocks of that layout (ceil(M / 128))
  };

  struct State {
    uint32_t cnt;   // chunks processed by this warp (selects the staging buffer)
    uint4 pre[4];   // prefetched input: 32 bf16 of this thread's row
    int pre_row, pre_col;  // which chunk `pre` holds (pre_col < 0: none)
  };

  __device__ static void init_state(State& s) {
    s.cnt = 0;
    s.pre_row = 0;
    s.pre_col = -1;
  }

  __device__ static __forceinline__ void load_chunk(const Params& ep, int M, int N, int row, int col,
                                                    uint4 (&v)[4]) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[j] = make_uint4(0, 0, 0, 0);
      if (ep.in != nullptr && row < M && col + j * 8 < N)
        v[j] = __ldg(reinterpret_cast<const uint4*>(ep.in + static_cast<size_t>(row) * N + col + j * 8));
    }
  }

  template <int BN>
  __device__ static bool tile(const Params& ep, const TileCtx& c, State& st, const WaitCtx& w) {
    static_assert(BN == 256, "partials are kept per 128-column half of a 256-column tile");
    const int col0 = c.nb * BN + c.cbeg;  // first column of this warp's share of the tile
    const int row = c.row0 + c.lane;
    int nch = (c.N - col0 + 63) / 64;
    if (nch > (c.cend - c.cbeg) / 64) nch = (c.cend - c.cbeg) / 64;
    if (nch < 0) nch = 0;
    const bool rows_live = c.row0 < c.M;
    float rs = 1.f;
    if (MODE == 1) rs = (row < c.M) ? __ldg(ep.r + row) : 0.f;
    float asc = 1.f, inv_s = 1.f, amx = 0.f;
    if (MODE >= 2) asc = __ldg(ep.sa) * __ldg(ep.sb);
    if (MODE == 2) inv_s = 1.0f / __ldg(ep.s_out);

    if (st.pre_col != col0 || st.pre_row != row) load_chunk(ep, c.M, c.N, row, col0, st.pre);
    // Row sums: each 64-column chunk from zero, the chunks of the tile's first
    // and second halves added in order, then the halves: the same rounding
    // whether one warp or two cover the tile.
    float ss_lo = 0.f, ss_hi = 0.f;
    for (int ch = 0; ch < nch; ++ch) {
      const int cc = col0 + ch * 64;
      float ss = 0.f;
      const int b = kNBuf == 2 ? static_cast<int>(st.cnt & 1) : 0;
      uint8_t* R = c.wsmem + b * kBufBytes;
      uint8_t* G = R + 4096;
      if (c.lane == 0) {
        if (kNBuf == 2)
          bulk_wait_read<1>();  // buffer b was last stored two chunks ago
        else
          bulk_wait_read<0>();
      }
      __syncwarp();
      uint32_t q8lo = 0, q8hi = 0;  // MODE 2: codes of the even j, stored with the odd j
      // the chunk's accumulator in two 32-column loads (fewer live registers)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
      uint4 cur[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) cur[u] = st.pre[u];
      // request the next 32 input columns (of this tile, or the first of the next tile)
      if (hh == 0 || ch + 1 < nch) {
        const int nc = cc + (hh + 1) * 32;
        load_chunk(ep, c.M, c.N, row, nc, st.pre);
        st.pre_row = row;
        st.pre_col = nc;
      } else if (c.has_next) {
        // (with eight warps the next tile has the same split of columns; a
        // half-tile unit is the last unit of its CTA pair)
        const int nrow = c.nrow0 + c.lane;
        load_chunk(ep, c.M, c.N, nrow, c.ncol0 + c.cbeg, st.pre);
        st.pre_row = nrow;
        st.pre_col = c.ncol0 + c.cbeg;
      } else {
        st.pre_col = -1;
      }
      uint32_t v[32];
      tmem_ld32(c.taddr + c.cbeg + ch * 64 + hh * 32, v);
      tmem_ld_wait(v);
      if constexpr (MODE == 3) {
        // one MXFP8 block: these 32 columns of this thread's row
        float g[32];
        float bmax = 0.f;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int j = hh * 4 + jj;
          const uint4 g4 = __ldg(reinterpret_cast<const uint4*>(ep.gamma + cc + j * 8));
          const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w};
          const uint32_t inw[4] = {cur[jj].x, cur[jj].y, cur[jj].z, cur[jj].w};
          uint32_t o1[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float h0 = fmaf(__uint_as_float(v[jj * 8 + 2 * e]), asc, bf16lo(inw[e]));
            const float h1 = fmaf(__uint_as_float(v[jj * 8 + 2 * e + 1]), asc, bf16hi(inw[e]));
            ss = fmaf(h0, h0, ss);
            ss = fmaf(h1, h1, ss);
            o1[e] = pack_bf16x2(h0, h1);
            g[jj * 8 + 2 * e] = h0 * bf16lo(gw[e]);
            g[jj * 8 + 2 * e + 1] = h1 * bf16hi(gw[e]);
            bmax = fmaxf(bmax, fmaxf(fabsf(g[jj * 8 + 2 * e]), fabsf(g[jj * 8 + 2 * e + 1])));
          }
          st_shared_v4(R + sw128_off(c.lane, j), make_uint4(o1[0], o1[1], o1[2], o1[3]));
        }
        const int ex = mx_e4m3_exponent(bmax);
        const float inv = exp2_neg(ex);
        uint32_t qw[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          qw[k] = pack_e4m3x2(g[4 * k] * inv, g[4 * k + 1] * inv) |
                  (pack_e4m3x2(g[4 * k + 2] * inv, g[4 * k + 3] * inv) << 16);
        // the block's 32 codes are 16-byte units 2 hh and 2 hh + 1 of the chunk's 64
        const uint4 u0 = make_uint4(qw[0], qw[1], qw[2], qw[3]);
        const uint4 u1 = make_uint4(qw[4], qw[5], qw[6], qw[7]);
        if (c.cend - c.cbeg == 64) {
          st_shared_v4(G + c.lane * 64 + (2 * hh) * 16, u0);
          st_shared_v4(G + c.lane * 64 + (2 * hh + 1) * 16, u1);
        } else {
          st_shared_v4(G + sw128_off(c.lane, (ch & 1) * 4 + 2 * hh), u0);
          st_shared_v4(G + sw128_off(c.lane, (ch & 1) * 4 + 2 * hh + 1), u1);
        }
        if (row < ep.sf_rb * 128)  // rows past M (zero) get e = 0: scale 1, as padding
          ep.sf_out[mx_sf_offset_a(row, (cc + hh * 32) >> 5, ep.sf_rb)] = static_cast<uint8_t>(ex + 127);
        continue;
      }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int j = hh * 4 + jj;
        const uint32_t off = sw128_off(c.lane, j);
        const uint32_t inw[4] = {cur[jj].x, cur[jj].y, cur[jj].z, cur[jj].w};
        uint32_t o1[4];
        if (MODE == 2) {
          const uint4 g4 = cc + j * 8 < c.N ? __ldg(reinterpret_cast<const uint4*>(ep.gamma + cc + j * 8))
                                            : make_uint4(0, 0, 0, 0);
          const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w};
          uint32_t q[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float h0 = fmaf(__uint_as_float(v[jj * 8 + 2 * e]), asc, bf16lo(inw[e]));
            const float h1 = fmaf(__uint_as_float(v[jj * 8 + 2 * e + 1]), asc, bf16hi(inw[e]));
            ss = fmaf(h0, h0, ss);
            ss = fmaf(h1, h1, ss);
            o1[e] = pack_bf16x2(h0, h1);
            const float g0 = h0 * bf16lo(gw[e]);
            const float g1 = h1 * bf16hi(gw[e]);
            amx = fmaxf(amx, fmaxf(fabsf(g0), fabsf(g1)));
            q[e] = pack_e4m3x2(g0 * inv_s, g1 * inv_s);
          }
          // 8 codes per j; two j make one 16-byte unit of the 128-column e4m3 row
          // (of a plain 64-column row when the warp covers 64 columns)
          const uint32_t lo = q[0] | (q[1] << 16), hi = q[2] | (q[3] << 16);
          if (j & 1) {
            if (c.cend - c.cbeg == 64)
              st_shared_v4(G + c.lane * 64 + (j >> 1) * 16, make_uint4(q8lo, q8hi, lo, hi));
            else
              st_shared_v4(G + sw128_off(c.lane, (ch & 1) * 4 + (j >> 1)), make_uint4(q8lo, q8hi, lo, hi));
          } else {
            q8lo = lo;
            q8hi = hi;
          }
        } else if (MODE == 0) {
          uint32_t o2[4];
          uint4 g4 = make_uint4(0, 0, 0, 0);  // gamma absent: hg is neither formed nor stored
          if (ep.gamma != nullptr && cc + j * 8 < c.N)
            g4 = __ldg(reinterpret_cast<const uint4*>(ep.gamma + cc + j * 8));
          const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float h0 = __uint_as_float(v[jj * 8 + 2 * e]) + bf16lo(inw[e]);
            const float h1 = __uint_as_float(v[jj * 8 + 2 * e + 1]) + bf16hi(inw[e]);
            ss = fmaf(h0, h0, ss);
            ss = fmaf(h1, h1, ss);
            o1[e] = pack_bf16x2(h0, h1);
            o2[e] = pack_bf16x2(h0 * bf16lo(gw[e]), h1 * bf16hi(gw[e]));
          }
          st_shared_v4(G + off, make_uint4(o2[0], o2[1], o2[2], o2[3]));
        } else {
          float dg[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float p0 = __uint_as_float(v[jj * 8 + 2 * e]);
            const float p1 = __uint_as_float(v[jj * 8 + 2 * e + 1]);
            const float g0 = bf16lo(inw[e]);
            const float g1 = bf16hi(inw[e]);
            ss = fmaf(g0, p0, ss);
            ss = fmaf(g1, p1, ss);
            o1[e] = pack_bf16x2(rs * g0, rs * g1);
            dg[2 * e] = rs * p0;
            dg[2 * e + 1] = rs * p1;
          }
          // fp32 columns j*8 .. j*8+7 live in box j/4, 16-byte chunks 2*(j%4) and 2*(j%4)+1
          uint8_t* Gb = G + (j >> 2) * 4096;
          st_shared_v4(Gb + sw128_off(c.lane, 2 * (j & 3)),
                       make_uint4(__float_as_uint(dg[0]), __float_as_uint(dg[1]), __float_as_uint(dg[2]),
                                  __float_as_uint(dg[3])));
          st_shared_v4(Gb + sw128_off(c.lane, 2 * (j & 3) + 1),
                       make_uint4(__float_as_uint(dg[4]), __float_as_uint(dg[5]), __float_as_uint(dg[6]),
                                  __float_as_uint(dg[7])));
        }
        st_shared_v4(R + off, make_uint4(o1[0], o1[1], o1[2], o1[3]));
      }
      }
      fence_async_smem();
      __syncwarp();
      if (c.lane == 0 && rows_live) {
        if (ep.has_out1 && c.khalf <= 0) tma_store_2d(&ep.tmOut1, R, cc, c.row0);
        if (ep.has_out2) {
          if (MODE >= 2) {
            // the e4m3 row holds two chunks: store after the odd one (or a lone last one);
            // a warp's 64 columns of a half tile go out as their own 64-byte rows
            if (c.cend - c.cbeg == 64)
              tma_store_2d(&ep.tmOut2h, G, col0, c.row0);
            else if ((ch & 1) || ch + 1 == nch)
              tma_store_2d(&ep.tmOut2, G, col0 + (ch & ~1) * 64, c.row0);
          } else if (MODE == 1 && c.khalf >= 0) {
            tma_reduce_add_2d(&ep.tmOut2, G, cc, c.row0);
            if (cc + 32 < c.N) tma_reduce_add_2d(&ep.tmOut2, G + 4096, cc + 32, c.row0);
          } else {
            tma_store_2d(&ep.tmOut2, G, cc, c.row0);
            if (MODE == 1 && cc + 32 < c.N) tma_store_2d(&ep.tmOut2, G + 4096, cc + 32, c.row0);
          }
        }
      }
      if (c.lane == 0) bulk_commit();
      ++st.cnt;
      if ((c.cbeg >> 6) + ch < (BN >> 7))
        ss_lo += ss;
      else
        ss_hi += ss;
    }
    // One partial per 128-column slot: slot 2 nb holds the tile's first half,
    // slot 2 nb + 1 its second half (when it starts inside N).  Whichever warp,
    // or half-tile unit, covers a half writes its slot, so halves computed by
    // different warps or CTA pairs need no hand-over.
    if (c.xchg != nullptr) {
      // a half tile over eight warps: this warp holds 64 of its slot's 128
      // columns; the second warp of the lane quarter hands its sums to the first
      const float mine = ss_lo + ss_hi;  // one of the two is zero
      const int slot = 2 * c.nb + (c.cbeg >= BN / 2 ? 1 : 0);
      if (c.half == 1) {
        c.xchg[c.lane] = mine;
        __syncwarp();
        if (c.lane == 0) mbar_arrive(c.xbar);
      } else {
        if (!__all_sync(0xffffffffu, mbar_wait(c.xbar, 0u, w))) return false;
        if (ep.partial != nullptr && row < c.M && slot * (BN / 2) < c.N)
          ep.partial[static_cast<size_t>(slot) * c.M + row] = mine + c.xchg[c.lane];
      }
    } else if (ep.partial != nullptr && row < c.M) {
      const int s0 = 2 * c.nb;
      float* p0 = ep.partial + static_cast<size_t>(s0) * c.M + row;
      float* p1 = p0 + c.M;
      const bool hi = c.cend > BN / 2 && (s0 + 1) * (BN / 2) < c.N;
      if (c.khalf >= 0) {
        // two K-halves add into a zeroed slot: 0 + a + b in either order
        if (c.cbeg < BN / 2) atomicAdd(p0, ss_lo);
        if (hi) atomicAdd(p1, ss_hi);
      } else {
        if (c.cbeg < BN / 2) *p0 = ss_lo;
        if (hi) *p1 = ss_hi;
      }
    }
    if (MODE == 2) {
      const unsigned m = __reduce_max_sync(0xffffffffu, __float_as_uint(amx));  // |hg| >= 0: bits order as values
      if (c.lane == 0 && m != 0u) atomicMax(ep.amax, m);
    }
    return true;
  }

  __device__ static void finish(const Params&, State&, uint64_t*, int lane, uint64_t) {
    if (lane == 0) bulk_wait_all<0>();
    __syncwarp();
  }
};

// ---------------------------------------------------------------------------
// Row-scaled bf16 output: out = r * acc (r null: out = acc).  The second GEMM
// of the block applies the RMSNorm row scale here.  With `partial` given, the
// epilogue also does the light reduction itself: each thread sums its row's
// T partial sums of squares (in the same order as the standalone reduction
// kernel) and forms r = 1 / sqrt(sum / N + eps); the tiles of column block 0
// write r out for the backward.
// ---------------------------------------------------------------------------
struct EpiRowScale {
  static constexpr int kSmemPerWarp = 2 * 4096;
  static constexpr int kBarsPerWarp = 0;
  static constexpr bool kPairedB = false;
  static constexpr bool kSplitN = true;

  struct Params {
    CUtensorMap tmOut;     // [M, N] bf16, box 64 x 32
    const float* r;        // [M] or null
    const float* partial;  // [T, M] partial sums of squares, or null
    int T;
    float inv_n, eps;
    float* r_out;          // [M] or null (written when partial is given)
    const float* sa;       // e4m3 operands: per-tensor scales of A and B (both null otherwise)
    const float* sb;
  };
  struct State {
    uint32_t cnt;
  };
  __device__ static void init_state(State& s) { s.cnt = 0; }

  // The row scale of this thread's row (0 past M).
  __device__ static __forceinline__ float row_scale(const Params& ep, const TileCtx& c, int row) {
    float rs = 1.f;
    if (ep.partial != nullptr) {
      rs = 0.f;
      if (row < c.M) {
        float sum = 0.f;
        // coherent (L2) loads: in the one-launch block the partials are written
        // by other CTAs of the same kernel.  Up to 16 slots are requested
        // together and then added in slot order (the order of the standalone
        // reduction kernel, so both give the same r).
        const float* pp = ep.partial + row;
        if (ep.T <= 16) {
          float pv[16];
#pragma unroll
          for (int t = 0; t < 16; ++t) pv[t] = t < ep.T ? __ldcg(pp + static_cast<size_t>(t) * c.M) : 0.f;
#pragma unroll
          for (int t = 0; t < 16; ++t)
            if (t < ep.T) sum += pv[t];
        } else {
          for (int t = 0; t < ep.T; ++t) sum += __ldcg(pp + static_cast<size_t>(t) * c.M);
        }
        rs = rsqrtf(sum * ep.inv_n + ep.eps);
        if (ep.r_out != nullptr && c.nb == 0 && c.cbeg == 0) ep.r_out[row] = rs;
      }
    } else if (ep.r != nullptr) {
      rs = (row < c.M) ? __ldg(ep.r + row) : 0.f;
    }
    return rs;
  }

  template <int BN>
  __device__ static bool tile(const Params& ep, const TileCtx& c, State& st, const WaitCtx&) {
    const int col0 = c.nb * BN + c.cbeg;  // first column of this unit (a half tile starts at 128)
    const int row = c.row0 + c.lane;
    int nch = (c.N - col0 + 63) / 64;
    if (nch > (c.cend - c.cbeg) / 64) nch = (c.cend - c.cbeg) / 64;
    float rs = row_scale(ep, c, row);
    if (ep.sa != nullptr) rs *= __ldg(ep.sa) * __ldg(ep.sb);  // dequantise with the row scale
    for (int ch = 0; ch < nch; ++ch) {
      uint8_t* O = c.wsmem + (st.cnt & 1) * 4096;
      if (c.lane == 0) bulk_wait_read<1>();
      __syncwarp();
      uint32_t v0[32], v1[32];
      tmem_ld64(c.taddr + c.cbeg + ch * 64, v0, v1);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          o[e] = pack_bf16x2(rs * acc_at(v0, v1, j * 8 + 2 * e), rs * acc_at(v0, v1, j * 8 + 2 * e + 1));
        st_shared_v4(O + sw128_off(c.lane, j), make_uint4(o[0], o[1], o[2], o[3]));
      }
      fence_async_smem();
      __syncwarp();
      if (c.lane == 0) {
        if (c.row0 < c.M) tma_store_2d(&ep.tmOut, O, col0 + ch * 64, c.row0);
        bulk_commit();
      }
      ++st.cnt;
    }
    return true;
  }

  __device__ static void finish(const Params&, State&, uint64_t*, int lane, uint64_t) {
    if (lane == 0) bulk_wait_all<0>();
    __syncwarp();
  }
};

// The second GEMM of the FP8 block: e4m3 A (hg8) and B (W2 stored [N2, K]),
// out = r * sa * sb * acc in bf16, with the light reduction folded in as in
// the bf16 block.
struct EpiRowScaleF8 : EpiRowScale {
  static constexpr bool kFp8 = true;
  static constexpr bool kSplitN = false;
};

// The second GEMM of the MXFP8 block: block-scaled A (hg) and B (W2 stored
// [N2, K]), out = r * acc in bf16 (the scales are applied inside the MMA),
// the light reduction folded in as in the bf16 block.  The tile has the only
// accumulator, so the epilogue first reads all of it into registers (bf16
// pairs, 128 per thread), releases it to the MMA, and only then stores the
// tile, chunk by chunk through one staging buffer: one 4 KB buffer per warp
// leaves the mainloop a stage more (261.9 against 266.5 us with two buffers
// and half of the tile staged before the release, both with three scale
// copies per k-block, on the 1B block's second GEMM).
struct EpiRowScaleMX : EpiRowScale {
  static constexpr int kSmemPerWarp = 4096;
  static constexpr bool kFp8 = true;
  static constexpr bool kMX = true;
  static constexpr bool kSplitN = false;

  __device__ static __forceinline__ void pack_chunk(uint32_t taddr, float rs, uint32_t (&o)[32]) {
    uint32_t v0[32], v1[32];
    tmem_ld64(taddr, v0, v1);
#pragma unroll
    for (int k = 0; k < 32; ++k) o[k] = pack_bf16x2(rs * acc_at(v0, v1, 2 * k), rs * acc_at(v0, v1, 2 * k + 1));
  }

  __device__ static __forceinline__ void stage_chunk(uint8_t* O, int lane, const uint32_t (&o)[32]) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      st_shared_v4(O + sw128_off(lane, j), make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]));
  }

  template <int BN>
  __device__ static bool tile(const Params& ep, const TileCtx& c, State&, const WaitCtx&) {
    static_assert(BN == 256, "four 64-column chunks per tile");
    const int col0 = c.nb * BN;
    const int row = c.row0 + c.lane;
    int nch = (c.N - col0 + 63) / 64;
    if (nch > 4) nch = 4;
    const float rs = row_scale(ep, c, row);
    uint32_t o0[32], o1[32], o2[32], o3[32];
    if (nch > 0) pack_chunk(c.taddr, rs, o0);
    if (nch > 1) pack_chunk(c.taddr + 64, rs, o1);
    if (nch > 2) pack_chunk(c.taddr + 128, rs, o2);
    if (nch > 3) pack_chunk(c.taddr + 192, rs, o3);
    // every tcgen05.ld of this warp has completed: hand the accumulator back
    tc_fence_before();
    __syncwarp();
    if (c.lane == 0) mbar_arrive_cluster(c.trel);
    const bool live = c.row0 < c.M;
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      if (ch < nch) {
        if (c.lane == 0) bulk_wait_read<0>();  // the buffer's last store has read it
        __syncwarp();
        stage_chunk(c.wsmem, c.lane, ch == 0 ? o0 : ch == 1 ? o1 : ch == 2 ? o2 : o3);
        fence_async_smem();
        __syncwarp();
        if (c.lane == 0) {
          if (live) tma_store_2d(&ep.tmOut, c.wsmem, col0 + ch * 64, c.row0);
          bulk_commit();
        }
      }
    }
    return true;
  }
};

// ---------------------------------------------------------------------------
// fp32 output (weight gradients): out = acc, or out = acc + out (accumulation
// over calls).  An optional correction serves the cross-entropy backward,
// whose gradient G is stored in bf16 and whose label entries' rounding
// residuals resid_i are kept in fp32: in dW_c = H^T G (output rows = hidden,
// columns = vocabulary), column v adds resid_i H[i, k] for every row i
// labelled v, in increasing i.  The rows come bucketed per 256-column
// vocabulary tile and sorted by (label, row), and are added to the staged
// tile in shared memory before it is stored.
// ---------------------------------------------------------------------------
struct EpiStoreF32 {
  static constexpr int kSmemPerWarp = 2 * 4096;
  static constexpr int kBarsPerWarp = 0;
  static constexpr bool kPairedB = false;
  static constexpr bool kSplitN = true;
  static constexpr bool kSplitK = true;  // out = acc is linear: K-halves add into a zeroed output

  struct Params {
    CUtensorMap tmOut;   // [M, N] fp32, box 32 x 32
    int add_to_out;      // 1: out += acc (accumulation over calls, a TMA reduce-add); 0: out = acc
    const float* fix_resid;            // [tokens] label-entry residuals
    long long fix_col0;                // vocabulary index of this chunk's column 0
    const int* fix_start;              // [tiles + 1] bucket offsets, or null (no correction)
    const int2* fix_entries;           // (label, row) sorted within each bucket
    const __nv_bfloat16* fix_H;        // [tokens, M]: the hidden states
    int fix_tile0;                     // bucket of this chunk's column 0 (chunk start / 256)
  };
  struct State {
    uint32_t cnt;
  };
  __device__ static void init_state(State& s) { s.cnt = 0; }

  template <int BN>
  __device__ static bool tile(const Params& ep, const TileCtx& c, State& st, const WaitCtx&) {
    static_assert(BN <= 256 && 256 % BN == 0, "a tile lies within one 256-column label bucket");
    const int col0 = c.nb * BN + c.cbeg;  // first column of this unit (a half tile starts at 128)
    const int row = c.row0 + c.lane;
    int nch = (c.N - col0 + 31) / 32;
    if (nch > (c.cend - c.cbeg) / 32) nch = (c.cend - c.cbeg) / 32;
    // this tile's run of (label, row) entries
    int e0 = 0, e1 = 0;
    if (ep.fix_start != nullptr && nch > 0) {
      const int bkt = ep.fix_tile0 + col0 / 256;
      e0 = ep.fix_start[bkt];
      e1 = ep.fix_start[bkt + 1];
    }
    // The run is fetched 32 entries at a time: lane l holds entry e0 + l, its
    // residual, and (for its own output row) H[row of entry j, row] for every
    // j of the batch, so the whole batch costs three rounds of loads.
    int2 fe = make_int2(-1, 0);
    float fr = 0.f;
    float hv[32];
    int nfe = 0;
    auto fetch_batch = [&](int first) {
      nfe = min(32, e1 - first);
      fe = make_int2(-1, 0);
      fr = 0.f;
      if (c.lane < nfe) {
        fe = ep.fix_entries[first + c.lane];
        fr = ep.fix_resid[fe.y];
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int tok = __shfl_sync(0xffffffffu, fe.y, j);
        hv[j] = (j < nfe && row < c.M) ? __bfloat162float(ep.fix_H[static_cast<size_t>(tok) * c.M + row]) : 0.f;
      }
    };
    if (e0 < e1) fetch_batch(e0);
    for (int ch = 0; ch < nch; ++ch) {
      const int cc = col0 + ch * 32;
      uint8_t* O = c.wsmem + (st.cnt & 1) * 4096;
      if (c.lane == 0) bulk_wait_read<1>();
      __syncwarp();
      uint32_t v[32];
      tmem_ld32(c.taddr + c.cbeg + ch * 32, v);
      tmem_ld_wait(v);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        st_shared_v4(O + sw128_off(c.lane, j), make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
      // entries are sorted by label, so the batch's entries of this 32-column
      // chunk are consecutive; add them in order (all branches warp-uniform).
      while (e0 < e1) {
        const long long vbase = ep.fix_col0 + cc;  // vocabulary index of this chunk's column 0
        int done = 0;  // entries of the batch left of the next chunk
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (j >= nfe) break;
          const long long q = static_cast<long long>(__shfl_sync(0xffffffffu, fe.x, j)) - vbase;
          if (q >= 32) break;
          ++done;
          const float rj = __shfl_sync(0xffffffffu, fr, j);
          if (q >= 0 && row < c.M) {
            float* sp = reinterpret_cast<float*>(O + sw128_off(c.lane, static_cast<int>(q >> 2))) + (q & 3);
            *sp += rj * hv[j];
          }
        }
        if (done < nfe) break;      // the rest of the batch lies right of this chunk
        e0 += nfe;                  // batch used up: fetch the next one
        if (e0 < e1) fetch_batch(e0);
      }
      fence_async_smem();
      __syncwarp();
      if (c.lane == 0) {
        if (c.row0 < c.M) {
          if (ep.add_to_out || c.khalf >= 0)
            tma_reduce_add_2d(&ep.tmOut, O, cc, c.row0);
          else
            tma_store_2d(&ep.tmOut, O, cc, c.row0);
        }
        bulk_commit();
      }
      ++st.cnt;
    }
    return true;
  }

  __device__ static void finish(const Params&, State&, uint64_t*, int lane, uint64_t) {
    if (lane == 0) bulk_wait_all<0>();
    __syncwarp();
  }
};

// ---------------------------------------------------------------------------
// SwiGLU: the accumulator of one tile holds [gate 128 | up 128] columns for
// output columns nb*128 .. nb*128+127 (the B operand is loaded as two halves,
// gate columns from W_gu[:, :F] and up columns from W_gu[:, F:]).
//   g = r * acc_gate, u = r * acc_up, act = silu(g) * u;
//   optionally g and u (bf16) are saved for the backward.
// ---------------------------------------------------------------------------
// kSave: gate and up are also kept (for the backward).  Without them the
// epilogue needs only the act double buffer, which leaves the mainloop a
// sixth stage.
template <bool kSave>
struct EpiSwiGLUT {
  static constexpr int kSmemPerWarp = kSave ? 2 * 4096 + 8192 : 2 * 4096;  // act double buffer (+ save buffer)
  static constexpr int kBarsPerWarp = 0;
  static constexpr bool kPairedB = true;

  struct Params {
    CUtensorMap tmAct;    // [M, F] bf16, box 64 x 32
    CUtensorMap tmSaveG;  // gate view of the [M, 2F] save tensor, box 64 x 32
    CUtensorMap tmSaveU;  // up view of the [M, 2F] save tensor, box 64 x 32
    const float* r;       // [M] or null
  };
  struct State {
    uint32_t cnt;
  };
  __device__ static void init_state(State& s) { s.cnt = 0; }

  __device__ static __forceinline__ float silu(float g) { return g / (1.0f + __expf(-g)); }

  template <int BN>
  __device__ static bool tile(const Params& ep, const TileCtx& c, State& st, const WaitCtx&) {
    constexpr int kHalf = BN / 2;  // output columns per tile
    const int ocol0 = c.nb * kHalf;
    const int row = c.row0 + c.lane;
    int nch = (c.N - ocol0 + 63) / 64;  // c.N = F here
    if (nch > kHalf / 64) nch = kHalf / 64;
    float rs = 1.f;
    if (ep.r != nullptr) rs = (row < c.M) ? __ldg(ep.r + row) : 0.f;
    constexpr bool save = kSave;
    uint8_t* SG = c.wsmem + 2 * 4096;
    uint8_t* SU = SG + 4096;
    for (int ch = 0; ch < nch; ++ch) {
      uint8_t* O = c.wsmem + (st.cnt & 1) * 4096;
      if (c.lane == 0) {
        if (save)
          bulk_wait_read<0>();
        else
          bulk_wait_read<1>();
      }
      __syncwarp();
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t vg[32], vu[32];
        tmem_ld32(c.taddr + ch * 64 + hh * 32, vg);
        tmem_ld32(c.taddr + kHalf + ch * 64 + hh * 32, vu);
        tmem_ld_wait(vg);
        reg_pin(vu);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          uint32_t o[4], og[4], ou[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = jj * 8 + 2 * e;
            const float g0 = rs * __uint_as_float(vg[i]), g1 = rs * __uint_as_float(vg[i + 1]);
            const float u0 = rs * __uint_as_float(vu[i]), u1 = rs * __uint_as_float(vu[i + 1]);
            o[e] = pack_bf16x2(silu(g0) * u0, silu(g1) * u1);
            og[e] = pack_bf16x2(g0, g1);
            ou[e] = pack_bf16x2(u0, u1);
          }
          const uint32_t off = sw128_off(c.lane, hh * 4 + jj);
          st_shared_v4(O + off, make_uint4(o[0], o[1], o[2], o[3]));
          if (save) {
            st_shared_v4(SG + off, make_uint4(og[0], og[1], og[2], og[3]));
            st_shared_v4(SU + off, make_uint4(ou[0], ou[1], ou[2], ou[3]));
          }
        }
      }
      fence_async_smem();
      __syncwarp();
      if (c.lane == 0) {
        if (c.row0 < c.M) {
          tma_store_2d(&ep.tmAct, O, ocol0 + ch * 64, c.row0);
          if (save) {
            tma_store_2d(&ep.tmSaveG, SG, ocol0 + ch * 64, c.row0);
            tma_store_2d(&ep.tmSaveU, SU, ocol0 + ch * 64, c.row0);
          }
        }
        bulk_commit();
      }
      ++st.cnt;
    }
    return true;
  }

  __device__ static void finish(const Params&, State&, uint64_t*, int lane, uint64_t) {
    if (lane == 0) bulk_wait_all<0>();
    __syncwarp();
  }
};
using EpiSwiGLU = EpiSwiGLUT<true>;     // act, gate and up
using EpiSwiGLUAct = EpiSwiGLUT<false>;  // act only

// ---------------------------------------------------------------------------
// SwiGLU backward in the down projection's dA GEMM: acc = d_act = d_out W_down^T
// for output columns j of this tile; with the saved gate g and up u of the same
// columns,
//   d_gate = d_act * u * silu'(g),  d_up = d_act * silu(g)
// (silu'(g) = s (1 + g (1 - s)), s = 1 / (1 + exp(-g))) are written to the
// [M, 2F] gradient (gate half, up half).  d_act never reaches memory.
// Each warp streams its 32 rows of g and u through two shared-memory buffers,
// one 64-column chunk (4 KB of g + 4 KB of u, 128-byte swizzle) per buffer,
// brought in by TMA one chunk ahead (the next tile's first chunk during this
// tile's last); d_gate and d_up overwrite the chunk in place and leave by TMA
// store.  g, u and the gradient are each touched once: their loads and
// stores carry the L2 evict-first policy, which keeps the GEMM operands (read
// again by every column block) in L2: 214 against 226 us on the 8192-token
// 1B MLP (8192 x 8192 x 2048), 442 against 525 MB read from DRAM.
// ---------------------------------------------------------------------------
struct EpiSwiGLUBwd {
  static constexpr int kSmemPerWarp = 2 * 8192;
  static constexpr int kBarsPerWarp = 2;  // per buffer: its g / u load has landed
  static constexpr bool kPairedB = false;

  struct Params {
    CUtensorMap tmG;   // gate view of the saved [M, 2F] (columns [0, F)), row stride 2F, box 64 x 32
    CUtensorMap tmU;   // up view (columns [F, 2F))
    CUtensorMap tmDG;  // gate view of d_gateup [M, F], row stride 2F, box 64 x 32
    CUtensorMap tmDU;  // up view of d_gateup
  };
  struct State {
    uint32_t used;    // chunks this warp has computed
    uint32_t issued;  // chunks whose g / u load this warp has issued (used or used + 1)
  };
  __device__ static void init_state(State& s) {
    s.used = 0;
    s.issued = 0;
  }

  // Lane 0 loads g and u of chunk number k of this warp (columns [col, col + 64)
  // of rows [row0, row0 + 32); out-of-range parts read as zero) into buffer
  // k & 1.  That buffer was last read by the stores of chunk k - 2, the latest
  // stores committed: wait until every committed store has read its data.
  __device__ static __forceinline__ void issue(const Params& ep, const TileCtx& c, uint32_t k, int col, int row0) {
    if (c.lane == 0) {
      bulk_wait_read<0>();
      uint8_t* buf = c.wsmem + (k & 1) * 8192;
      uint64_t* bar = c.wbars + (k & 1);
      const uint64_t pol = l2_evict_first_policy();
      mbar_arrive_expect_tx(bar, 8192);
      tma_load_2d_hint(buf, &ep.tmG, bar, col, row0, pol);
      tma_load_2d_hint(buf + 4096, &ep.tmU, bar, col, row0, pol);
    }
  }

  template <int BN>
  __device__ static bool tile(const Params& ep, const TileCtx& c, State& st, const WaitCtx& w) {
    const int col0 = c.nb * BN;
    int nch = (c.N - col0 + 63) / 64;
    if (nch > BN / 64) nch = BN / 64;
    if (st.issued == st.used) issue(ep, c, st.issued++, col0, c.row0);  // nothing prefetched yet
    for (int ch = 0; ch < nch; ++ch) {
      const uint32_t k = st.used;
      // the next chunk: this tile's, else the first of this warp's next tile
      if (ch + 1 < nch)
        issue(ep, c, st.issued++, col0 + (ch + 1) * 64, c.row0);
      else if (c.has_next)
        issue(ep, c, st.issued++, c.ncol0, c.nrow0);
      if (!__all_sync(0xffffffffu, mbar_wait(c.wbars + (k & 1), (k >> 1) & 1u, w))) return false;
      uint8_t* G = c.wsmem + (k & 1) * 8192;
      uint8_t* U = G + 4096;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t v[32];
        tmem_ld32(c.taddr + ch * 64 + hh * 32, v);
        tmem_ld_wait(v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t off = sw128_off(c.lane, hh * 4 + j);
          const uint4 gq = ld_shared_v4(G + off);
          const uint4 uq = ld_shared_v4(U + off);
          const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w};
          const uint32_t uw[4] = {uq.x, uq.y, uq.z, uq.w};
          uint32_t og[4], ou[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float dg2[2], du2[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float da = __uint_as_float(v[j * 8 + 2 * e + h]);
              const float g = h ? bf16hi(gw[e]) : bf16lo(gw[e]);
              const float u = h ? bf16hi(uw[e]) : bf16lo(uw[e]);
              const float sg = __fdividef(1.0f, 1.0f + __expf(-g));  // sigmoid; 0 when exp overflows
              dg2[h] = da * u * (sg * (1.0f + g * (1.0f - sg)));
              du2[h] = da * (g * sg);
            }
            og[e] = pack_bf16x2(dg2[0], dg2[1]);
            ou[e] = pack_bf16x2(du2[0], du2[1]);
          }
          st_shared_v4(G + off, make_uint4(og[0], og[1], og[2], og[3]));
          st_shared_v4(U + off, make_uint4(ou[0], ou[1], ou[2], ou[3]));
        }
      }
      fence_async_smem();
      __syncwarp();
      if (c.lane == 0) {
        if (c.row0 < c.M) {
          const uint64_t pol = l2_evict_first_policy();
          tma_store_2d_hint(&ep.tmDG, G, col0 + ch * 64, c.row0, pol);
          tma_store_2d_hint(&ep.tmDU, U, col0 + ch * 64, c.row0, pol);
        }
        bulk_commit();
      }
      ++st.used;
    }
    return true;
  }

  // A load issued for a chunk that was never computed (only after a failed
  // wait ended the tile loop) lands before the CTA's shared memory is freed;
  // the wait is bounded like every other.
  __device__ static void finish(const Params&, State& st, uint64_t* wbars, int lane, uint64_t wait_ns) {
    if (st.issued != st.used) {
      const uint32_t k = st.used;
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(wbars + (k & 1), (k >> 1) & 1u) && globaltimer_ns() - t0 < wait_ns) {
      }
    }
    if (lane == 0) bulk_wait_all<0>();
    __syncwarp();
  }
};

// ---------------------------------------------------------------------------
// LM-head cross-entropy: block log-sum-exp of the tile with an online
// (running max, running sum-exp) state over 32-column chunks.  Logits stay in
// fp32 registers and never reach memory.  Per (column tile, row) the tile's
// (max, sum-exp) goes to the workspace; the tile that holds a row's label
// also writes that logit.  A combine kernel merges the tiles.
// ---------------------------------------------------------------------------
struct EpiCE {
  static constexpr int kSmemPerWarp = 0;
  static constexpr int kBarsPerWarp = 0;
  static constexpr bool kPairedB = false;

  struct Params {
    float* ws_m;            // [n_tiles_v, M] tile max
    float* ws_s;            // [n_tiles_v, M] tile sum of exp(z - max)
    float* zlab;            // [M] label logit
    const int64_t* labels;  // [M]
    const float* r;         // [M] or null (row scale of a preceding RMSNorm)
  };
  struct State {
    int unused;
  };
  __device__ static void init_state(State&) {}

  template <int BN>
  __device__ static bool tile(const Params& ep, const TileCtx& c, State&, const WaitCtx&) {
    constexpr float kL2E = 1.4426950408889634f;
    const int col0 = c.nb * BN;
    const int row = c.row0 + c.lane;
    const bool valid = row < c.M;
    const int V = c.N;
    long long lab = valid ? ep.labels[row] : -1;
    const float rs = (ep.r != nullptr && valid) ? __ldg(ep.r + row) : 1.f;
    float m = -INFINITY, s = 0.f, zl = 0.f;
    bool got = false;
    int nch = (V - col0 + 31) / 32;
    if (nch > BN / 32) nch = BN / 32;
    for (int ch = 0; ch < nch; ++ch) {
      const int cc = col0 + ch * 32;
      uint32_t v[32];
      tmem_ld32(c.taddr + ch * 32, v);
      tmem_ld_wait(v);
      float z[32];
      float cm = -INFINITY;
      const long long d = lab - cc;                                    // label position inside this chunk,
      const int dl = (d >= 0 && d < 32) ? static_cast<int>(d) : -1;   // if any
      const bool whole = cc + 32 <= V;                                 // no ragged columns in this chunk
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        z[e] = (whole || cc + e < V) ? rs * __uint_as_float(v[e]) : -INFINITY;
        cm = fmaxf(cm, z[e]);
        zl = (e == dl) ? z[e] : zl;
      }
      got = got || dl >= 0;
      const float mn = fmaxf(m, cm);
      const float base = mn * kL2E;
      float sum = 0.f;
#pragma unroll
      for (int e = 0; e < 32; ++e) sum += ex2_approx(fmaf(z[e], kL2E, -base));
      s = s * ex2_approx((m - mn) * kL2E) + sum;
      m = mn;
    }
    if (valid) {
      const size_t o = static_cast<size_t>(c.nb) * c.M + row;
      ep.ws_m[o] = m;
      ep.ws_s[o] = s;
      if (got) ep.zlab[row] = zl;
    }
    return true;
  }

  __device__ static void finish(const Params&, State&, uint64_t*, int, uint64_t) {}
};

// ---------------------------------------------------------------------------
// RoPE in the QKV projection's epilogue (rotate-half form).  For every head of
// head_dim columns that lies below rope_cols (the q and k heads), columns i and
// i + head_dim/2 form a pair rotated by the angle pos * theta^(-2 i / head_dim):
//   (a, b) -> (a cos - b sin, b cos + a sin);
// heads at or beyond rope_cols (v) are stored unrotated.  One thread owns one
// row, so both columns of every pair are in its registers.  The angle is taken
// in turns, pos * theta^(-2i/d) / (2 pi), in fp64 (the per-frequency factors
// come precomputed in the kernel parameters); only its fractional part goes
// to sincospif, so large positions keep their accuracy without a range
// reduction.  With head_dim 64 the sines and cosines of the row's 32
// frequencies are computed once per tile and reused for every head.  Each
// head is staged on its own (one or two 64-column boxes) and stored at once,
// so the staging takes 8 KB per warp and the mainloop keeps six stages.
// ---------------------------------------------------------------------------
struct EpiRope {
  // Four warps, each taking all the tile's columns (four heads of 64 or two
  // of 128), which leaves the mainloop a sixth stage: on the 1B QKV
  // projection 80.5 against 84.7 us with eight warps (64-wide heads), 88.4
  // against 92.1 us with 128-wide heads.  A half tile (the split last wave)
  // gives each warp 128 columns, whole heads either way.
  static constexpr int kWarps = 4;
  static constexpr int kSmemPerWarp = 8192;  // two 64-column x 32-row bf16 boxes
  static constexpr int kBarsPerWarp = 0;
  static constexpr bool kPairedB = false;
  static constexpr bool kSplitN = true;

  struct Params {
    CUtensorMap tmOut;      // [M, N] bf16, box 64 x 32
    const int* positions;   // [M]
    int head_dim;           // 64 or 128
    int rope_cols;          // columns [0, rope_cols) are rotated; a multiple of head_dim
    uint64_t turn_fx[64];   // theta^(-2i/head_dim) / (2 pi), i < head_dim / 2, in units of 2^-64 turn
  };
  struct State {
    uint32_t cnt;  // heads staged so far (alternates the two boxes when head_dim is 64)
  };
  __device__ static void init_state(State& s) { s.cnt = 0; }

  template <int BN>
  __device__ static bool tile(const Params& ep, const TileCtx& c, State& st, const WaitCtx&) {
    const int col0 = c.nb * BN + c.cbeg;  // first column of this warp's half of the tile
    const int row = c.row0 + c.lane;
    const int dh = ep.head_dim;
    const int half = dh >> 1;
    // the position as a 64-bit integer: pos x turn_fx mod 2^64 is the angle's
    // fraction of a turn, exact (two's complement keeps negative positions right)
    const uint64_t pos = (row < c.M) ? static_cast<uint64_t>(static_cast<int64_t>(ep.positions[row])) : 0u;
    int ncols = c.N - col0;
    if (ncols > c.cend - c.cbeg) ncols = c.cend - c.cbeg;
    const int nheads = ncols / dh;
    float cs[32], sn[32];
    for (int hd = 0; hd < nheads; ++hd) {
      const int hc0 = hd * dh;  // head's first column within this warp's half
      const bool rot = col0 + hc0 < ep.rope_cols;
      // head_dim 64: one box per head, two in turn; 128: both boxes per head
      uint8_t* S = c.wsmem + (dh == 64 ? (st.cnt & 1) * 4096 : 0);
      if (c.lane == 0) {
        if (dh == 64)
          bulk_wait_read<1>();  // this box was last stored two heads ago
        else
          bulk_wait_read<0>();
      }
      __syncwarp();
      for (int s = 0; s < half / 32; ++s) {
        if (rot && (dh != 64 || hd == 0 || col0 + (hd - 1) * dh >= ep.rope_cols)) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            // top 32 bits: the signed fraction of a turn in [-1/2, 1/2) x 2^32;
            // times 2^-31 it is the angle over pi, in [-1, 1)
            const uint64_t t = pos * ep.turn_fx[s * 32 + e];
            const float a = static_cast<float>(static_cast<int32_t>(static_cast<uint32_t>(t >> 32))) * 0x1p-31f;
            sincospif(a, &sn[e], &cs[e]);
          }
        }
        uint32_t va[32], vb[32];
        tmem_ld32(c.taddr + c.cbeg + hc0 + s * 32, va);
        tmem_ld32(c.taddr + c.cbeg + hc0 + half + s * 32, vb);
        tmem_ld_wait(va);
        reg_pin(vb);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t pa[4], pb[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            float oa[2], ob[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int e = q * 8 + 2 * e2 + h;
              const float a = __uint_as_float(va[e]);
              const float bb = __uint_as_float(vb[e]);
              oa[h] = rot ? a * cs[e] - bb * sn[e] : a;
              ob[h] = rot ? bb * cs[e] + a * sn[e] : bb;
            }
            pa[e2] = pack_bf16x2(oa[0], oa[1]);
            pb[e2] = pack_bf16x2(ob[0], ob[1]);
          }
          const int ca = s * 32 + q * 8;  // columns within the head
          const int cb = half + s * 32 + q * 8;
          st_shared_v4(S + (ca >> 6) * 4096 + sw128_off(c.lane, (ca & 63) >> 3),
                       make_uint4(pa[0], pa[1], pa[2], pa[3]));
          st_shared_v4(S + (cb >> 6) * 4096 + sw128_off(c.lane, (cb & 63) >> 3),
                       make_uint4(pb[0], pb[1], pb[2], pb[3]));
        }
      }
      fence_async_smem();
      __syncwarp();
      if (c.lane == 0) {
        if (c.row0 < c.M)
          for (int bx = 0; bx < dh / 64; ++bx) tma_store_2d(&ep.tmOut, S + bx * 4096, col0 + hc0 + bx * 64, c.row0);
        bulk_commit();
      }
      ++st.cnt;
    }
    return true;
  }

  __device__ static void finish(const Params&, State&, uint64_t*, int lane, uint64_t) {
    if (lane == 0) bulk_wait_all<0>();
    __syncwarp();
  }
};

// ---------------------------------------------------------------------------
// Cross-entropy backward, block-local: the logits of one vocabulary chunk are
// recomputed in the accumulator and, with the forward's saved log-sum-exp,
// turned into the gradient
//   G_ij = d_i (exp(z_ij - lse_i) - [col0 + j == label_i]),   z = r_i (H W_chunk)_ij
// (d_i = d_loss_i, or `scale` for every token when d_loss is null), stored in
// bf16 for the two GEMMs that consume the chunk (dH += G W_chunk^T and
// dW_chunk = H^T G).  The logits themselves are never stored.
// ---------------------------------------------------------------------------
struct EpiCEGrad {
  static constexpr int kSmemPerWarp = 2 * 4096;
  static constexpr int kBarsPerWarp = 0;
  static constexpr bool kPairedB = false;
  static constexpr bool kHasPre = true;

  struct Params {
    CUtensorMap tmG;        // [M, Vc] bf16, box 64 x 32
    const int64_t* labels;  // [M]
    const float* lse;       // [M] from the forward
    const float* d_loss;    // [M] or null
    const float* r;         // [M] or null
    float scale;            // weight of every token when d_loss is null (1/M: the mean)
    float* resid;           // [M]: G - bf16(G) at each row's label entry (or null)
    long long col_offset;   // vocabulary index of this chunk's column 0
    // The previous chunk's exact label entries of dH (dH[i, :] += resid_i
    // W[:, label_i] over its label buckets [fix_b0, fix_b1)), added by the
    // epilogue warps of every CTA before their first tile, while its mainloop
    // runs; fix_start null: nothing to add.  Launched after the previous
    // chunk's dH GEMM, so that one has completed (griddepcontrol.wait).
    const int2* fix_entries;
    const int* fix_start;
    int fix_b0, fix_b1;
    const __nv_bfloat16* fix_W;
    long long fix_V;
    int fix_K;
    float* fix_dH;
  };
  struct State {
    uint32_t cnt;
  };
  __device__ static void init_state(State& s) { s.cnt = 0; }

  __device__ static void pre(const Params& ep, long long warp, long long nwarps, int lane) {
    if (ep.fix_start != nullptr)
      ce_label_dh_fix_range(ep.fix_entries, ep.fix_start, ep.fix_b0, ep.fix_b1, ep.resid, ep.fix_W, ep.fix_V,
                            ep.fix_K, ep.fix_dH, warp, nwarps, lane);
  }

  template <int BN>
  __device__ static bool tile(const Params& ep, const TileCtx& c, State& st, const WaitCtx&) {
    constexpr float kL2E = 1.4426950408889634f;
    const int col0 = c.nb * BN;
    const int row = c.row0 + c.lane;
    const bool live = row < c.M;
    int nch = (c.N - col0 + 63) / 64;
    if (nch > BN / 64) nch = BN / 64;
    const float rs = (ep.r != nullptr && live) ? __ldg(ep.r + row) : 1.f;
    const float lse2 = live ? __ldg(ep.lse + row) * kL2E : 0.f;
    const float d = live ? (ep.d_loss != nullptr ? __ldg(ep.d_loss + row) : ep.scale) : 0.f;
    const long long lab = live ? ep.labels[row] - ep.col_offset : -1;
    for (int ch = 0; ch < nch; ++ch) {
      const int cc = col0 + ch * 64;
      const long long dd = lab - cc;                                    // label column inside this chunk,
      const int ll = (dd >= 0 && dd < 64) ? static_cast<int>(dd) : -1;  // if any
      float glab = 0.f;
      uint8_t* O = c.wsmem + (st.cnt & 1) * 4096;
      if (c.lane == 0) bulk_wait_read<1>();
      __syncwarp();
      uint32_t v0[32], v1[32];
      tmem_ld64(c.taddr + ch * 64, v0, v1);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float gg[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int jj = j * 8 + 2 * e + h;
            const float z = rs * acc_at(v0, v1, jj);
            const float p = ex2_approx(fmaf(z, kL2E, -lse2));
            float g = d * p;
            if (jj == ll) {
              g = d * (p - 1.0f);
              glab = g;
            }
            gg[h] = g;
          }
          o[e] = pack_bf16x2(gg[0], gg[1]);
        }
        st_shared_v4(O + sw128_off(c.lane, j), make_uint4(o[0], o[1], o[2], o[3]));
      }
      // the label entry dominates its dW column: keep what bf16 rounding drops
      if (ll >= 0 && ep.resid != nullptr) ep.resid[row] = glab - __bfloat162float(__float2bfloat16_rn(glab));
      fence_async_smem();
      __syncwarp();
      if (c.lane == 0) {
        if (c.row0 < c.M) tma_store_2d(&ep.tmG, O, cc, c.row0);
        bulk_commit();
      }
      ++st.cnt;
    }
    return true;
  }

  __device__ static void finish(const Params&, State&, uint64_t*, int lane, uint64_t) {
    if (lane == 0) bulk_wait_all<0>();
    __syncwarp();
  }
};

}  // namespace coda
