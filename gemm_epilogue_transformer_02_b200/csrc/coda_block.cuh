// The GEMM-RMSNorm-GEMM block as one persistent launch.
//
// KuCoin news flash "CODA: new research optimizes transformer training with
// GEMM epilogue programming", section "CODA: the secret in the epilogue": the
// first GEMM's epilogue adds the residual and emits partial sums of squares,
// a light reduction turns them into the RMSNorm row scale r, and the second
// GEMM applies r (a per-row scalar that commutes with the matmul) in its own
// epilogue.  Here both GEMMs run in one kernel over CTA pairs (tcgen05
// cta_group::2, 256 x 256 tiles):
//
//   tiles [0, n1)       first GEMM  (x W1 + res -> h, hg, partials), row-major
//                       order so that row blocks complete early;
//   tiles [n1, n1 + n2) second GEMM (r * (hg W2), r formed in its epilogue from
//                       the partials), in groups of `group2` row blocks, each
//                       group's row blocks for one column block after another,
//                       so that the first second-GEMM tiles need only the first
//                       row blocks of the first GEMM.
//
// Tiles are dealt round-robin to the resident clusters, so every cluster runs
// its first-GEMM tiles before any second-GEMM tile.  A first-GEMM tile's
// epilogue warps publish their finished rows with a release increment of the
// row block's counter once their TMA stores and partial sums are complete; a
// second-GEMM tile's producer (and its epilogue, before reading the partials)
// waits, bounded in time, until the counter shows all of that row block's
// first-GEMM tiles.  Only first-GEMM work is ever waited on and it never
// waits itself, so with all clusters resident the waits always end; the
// second GEMM's tiles fill the idle SMs of the first GEMM's last wave.
#pragma once

#include "coda_gemm.cuh"

namespace coda {

struct BlockParams {
  CUtensorMap tmA1;  // x [M, K1], K-major
  CUtensorMap tmB1;  // W1 [K1, N1], MN-major
  CUtensorMap tmA2;  // hg [M, N1], K-major
  CUtensorMap tmB2;  // W2 [N1, N2], MN-major
  EpiLoadStore2<0>::Params ep1;
  EpiRowScale::Params ep2;
  int* ready;        // [n_mt] completion counters (zero at launch)
  int M, K1, N1, N2;
  int n_mt, n_nt1, n_nt2, n1, n2;
  // the last nsplit second-GEMM tiles run as two 128-column halves each (a
  // last partial wave on at most half of the pairs becomes a wave of halves)
  int nsplit;
  int group2;        // row blocks per raster group of the second GEMM
  int ready_target;  // counter value of a finished row block: n_nt1 tiles x 2 CTAs x 4 warps
  uint64_t wait_ns;
};

struct BlockTile {
  int phase, mb, nb;
  int half;  // -1: a whole tile; 0 or 1: that 128-column half of a second-GEMM tile
};

__device__ __forceinline__ BlockTile block_tile(const BlockParams& p, int t) {
  BlockTile b;
  b.half = -1;
  if (t < p.n1) {
    b.phase = 0;
    b.mb = t / p.n_nt1;
    b.nb = t - b.mb * p.n_nt1;
  } else {
    int u = t - p.n1;
    const int s0 = p.n2 - p.nsplit;
    if (u >= s0) {
      b.half = (u - s0) & 1;
      u = s0 + ((u - s0) >> 1);
    }
    b.phase = 1;
    const int per_group = p.group2 * p.n_nt2;
    const int g = u / per_group;
    const int first = g * p.group2;
    const int gs = p.n_mt - first < p.group2 ? p.n_mt - first : p.group2;
    const int r = u - g * per_group;
    b.mb = first + r % gs;
    b.nb = r / gs;
  }
  return b;
}

template <int STAGES>
struct BlockSmem {
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = 128 * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kEpiPerWarp = EpiLoadStore2<0>::kSmemPerWarp > EpiRowScale::kSmemPerWarp
                                         ? EpiLoadStore2<0>::kSmemPerWarp
                                         : EpiRowScale::kSmemPerWarp;
  static constexpr int kEpiBytes = kEpiWarps * kEpiPerWarp;
  static constexpr int kNumBars = 2 * STAGES + 2 + 2 + 1;
  static constexpr int kBytes = 1024 + STAGES * kStageBytes + kEpiBytes + kNumBars * 8 + 16;
  static_assert(kEpiPerWarp % 1024 == 0, "per-warp epilogue buffers keep the 128-byte swizzle alignment");
};

template <int STAGES>
__global__ void __launch_bounds__(kThreads, 1) coda_block_kernel(const __grid_constant__ BlockParams p) {
  using S = BlockSmem<STAGES>;
  constexpr int BN = 256;
  constexpr int kTileM = 2 * kBM;
  constexpr int kBCols = BN / 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * S::kABytes;
  uint8_t* sEpi = smem + STAGES * S::kStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + S::kEpiBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int tile_step = static_cast<int>(gridDim.x >> 1);
  const int tile_first = static_cast<int>(blockIdx.x >> 1);
  const int ntiles = p.n1 + p.n2 + p.nsplit;  // schedule units

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmA1);
    tma_prefetch_desc(&p.tmB1);
    tma_prefetch_desc(&p.tmA2);
    tma_prefetch_desc(&p.tmB2);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, 2 * BN);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const WaitCtx w{abort_flag, p.wait_ns};
  const int nkb1 = (p.K1 + kBK - 1) / kBK;
  const int nkb2 = (p.N1 + kBK - 1) / kBK;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      const uint32_t full0 = mapa_shared(smem_u32(full), 0);
      for (int t = tile_first; ok && t < ntiles; t += tile_step) {
        const BlockTile bt = block_tile(p, t);
        const CUtensorMap* mA = bt.phase ? &p.tmA2 : &p.tmA1;
        const CUtensorMap* mB = bt.phase ? &p.tmB2 : &p.tmB1;
        const int nkb = bt.phase ? nkb2 : nkb1;
        if (bt.phase == 1) {
          // hg of this row block must be complete before the copies read it
          if (!counter_wait(p.ready + bt.mb, p.ready_target, w)) break;
          fence_proxy_async_global();
        }
        const int arow = bt.mb * kTileM + static_cast<int>(rank) * kBM;
        // a half tile: 64 B columns per CTA, starting at its half
        const int bcol = bt.half < 0 ? bt.nb * BN + static_cast<int>(rank) * kBCols
                                     : bt.nb * BN + bt.half * (BN / 2) + static_cast<int>(rank) * (kBCols / 2);
        const int nbox = bt.half < 0 ? kBCols / 64 : kBCols / 128;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, w)) {
            ok = false;
            break;
          }
          uint8_t* a = sA + stage * S::kABytes;
          uint8_t* b = sB + stage * S::kBBytes;
          if (rank == 0)
            mbar_arrive_expect_tx(&full[stage], bt.half < 0 ? 2 * S::kStageBytes : 2 * (S::kABytes + S::kBBytes / 2));
          const uint32_t fb = full0 + stage * 8;
          tma_load_2d_pair(a, mA, fb, kb * kBK, arow);
          for (int j = 0; j < nbox; ++j)
            tma_load_2d_pair(b + j * (64 * kBK * 2), mB, fb, bcol + j * 64, kb * kBK);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      const long n = issued < STAGES ? issued : STAGES;
      for (long i = 0; i < n; ++i) {
        if (stage == 0) {
          stage = STAGES - 1;
          phase ^= 1u;
        } else {
          --stage;
        }
        drain_wait(&empty[stage], phase, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0 && rank == 0) {
      constexpr uint32_t kIdesc = idesc_bf16_f32(kTileM, BN, false, true);
      constexpr uint32_t kIdescH = idesc_bf16_f32(kTileM, BN / 2, false, true);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int t = tile_first; ok && t < ntiles; t += tile_step, ++it) {
        const BlockTile bt = block_tile(p, t);
        const int nkb = bt.phase == 0 ? nkb1 : nkb2;
        const uint32_t idesc = bt.half < 0 ? kIdesc : kIdescH;
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], aph ^ 1u, w)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * BN + (bt.half > 0 ? BN / 2 : 0);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, w)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * S::kABytes);
          const uint32_t b0 = smem_u32(sB + stage * S::kBBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(a0 + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(b0 + kk * 16 * 128, 64 * kBK * 2, 1024);
            tc_mma_bf16_pair(d, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          tc_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(&tfull[acc], 0x3);
      }
      tc_commit_pair(drain);
      drain_wait(drain, 0, p.wait_ns);
    }
  } else {
    // --------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int ew = warp - 2;
    uint8_t* wsmem = sEpi + ew * S::kEpiPerWarp;
    const uint32_t tempty0 = mapa_shared(smem_u32(tempty), 0);
    EpiLoadStore2<0>::State st1;
    EpiRowScale::State st2;
    EpiLoadStore2<0>::init_state(st1);
    EpiRowScale::init_state(st2);
    bool in_phase2 = false;
    int it = 0;
    for (int t = tile_first; t < ntiles; t += tile_step, ++it) {
      const BlockTile bt = block_tile(p, t);
      const int acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph, w))) break;
      tc_fence_after();
      TileCtx c;
      c.M = p.M;
      c.mb = bt.mb;
      c.nb = bt.nb;
      c.row0 = bt.mb * kTileM + static_cast<int>(rank) * kBM + q * 32;
      c.taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN;
      c.lane = lane;
      c.wsmem = wsmem;
      c.wbars = nullptr;
      bool ok = true;
      if (bt.phase == 0) {
        c.N = p.N1;
        const int tn = t + tile_step;
        c.has_next = tn < p.n1;  // the input prefetch only crosses into first-GEMM tiles
        c.nrow0 = 0;
        c.ncol0 = 0;
        if (c.has_next) {
          const BlockTile nt = block_tile(p, tn);
          c.nrow0 = nt.mb * kTileM + static_cast<int>(rank) * kBM + q * 32;
          c.ncol0 = nt.nb * BN;
        }
        ok = EpiLoadStore2<0>::tile<BN>(p.ep1, c, st1, w);
      } else {
        c.N = p.N2;
        c.has_next = false;
        if (bt.half >= 0) {
          c.cbeg = bt.half * (BN / 2);
          c.cend = c.cbeg + BN / 2;
        }
        if (!in_phase2) {
          // the staging buffers change owners: the first GEMM's stores must have read them
          if (lane == 0) bulk_wait_read<0>();
          __syncwarp();
          in_phase2 = true;
        }
        // the partials of this row block are read by every lane: acquire them
        ok = __all_sync(0xffffffffu, counter_wait(p.ready + bt.mb, p.ready_target, w));
        if (ok) ok = EpiRowScale::tile<BN>(p.ep2, c, st2, w);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty0 + acc * 8);
      if (!ok) break;
      if (bt.phase == 0) {
        // publish this warp's rows of the tile: stores complete, partials visible
        if (lane == 0) {
          bulk_wait_all<0>();
          fence_proxy_async_global();
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) red_release_add(p.ready + bt.mb, 1);
      }
    }
    if (lane == 0) bulk_wait_all<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 2 * BN);
  }
}

}  // namespace coda
