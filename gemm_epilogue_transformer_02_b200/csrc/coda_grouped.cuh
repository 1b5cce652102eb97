// Two independent GEMMs in one persistent launch (CTA pairs, bf16).
//
// The backward passes of the KuCoin news flash "CODA: new research optimizes
// transformer training with GEMM epilogue programming" (section "CODA: the
// secret in the epilogue": the backward inherits the block-local structure)
// end in pairs of GEMMs that read the same gradient: dH and dW of a
// cross-entropy chunk, d_y and dW_gu of the SwiGLU MLP, dx and dW1 of the
// block.  Launched one after the other each ends in a partial wave (3.46 and
// 1.73 waves of 256 x 256 tiles on 74 CTA pairs for the cross-entropy pair);
// here both tile sets share one persistent grid.
//
// Scheduling is static and balanced: the tiles of problem 0 (the longer ones,
// more k-blocks per tile) go round-robin, and the tiles of problem 1 fill
// each pair up to a common makespan (`target`, in k-blocks, chosen on the
// host as the smallest that covers all tiles; see PairTiles).  Every warp of
// both CTAs of a pair derives the same list.
//
// The mainloop and the warp roles are those of coda_gemm_kernel (see
// coda_gemm.cuh); the operand layouts (K- or MN-major A and B) are runtime
// properties of each problem here, and each problem has its own epilogue.
#pragma once

#include "coda_gemm.cuh"

namespace coda {

template <class E0, class E1>
struct GroupedParams {
  CUtensorMap tmA[2];
  CUtensorMap tmB[2];
  typename E0::Params ep0;
  typename E1::Params ep1;
  int M[2], N[2], K[2];
  int n_mt[2], n_nt[2], group_m[2];
  int a_mn[2], b_mn[2];
  int ntiles[2];
  int target;  // makespan in k-blocks
  uint64_t wait_ns;
};

template <class E0, class E1>
struct GroupedSmem {
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = 128 * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kPerWarp = E0::kSmemPerWarp > E1::kSmemPerWarp ? E0::kSmemPerWarp : E1::kSmemPerWarp;
  static constexpr int kBarsPerWarp = E0::kBarsPerWarp > E1::kBarsPerWarp ? E0::kBarsPerWarp : E1::kBarsPerWarp;
  static constexpr int kEpiBytes = kEpiWarps * kPerWarp;
  template <int STAGES>
  static constexpr int bytes() {
    return 1024 + STAGES * kStageBytes + kEpiBytes + (2 * STAGES + 5 + kEpiWarps * kBarsPerWarp) * 8 + 16;
  }
  static_assert(kPerWarp % 1024 == 0, "per-warp epilogue buffers keep the 128-byte swizzle alignment");
  static_assert(epi_warps<E0>::value == 4 && epi_warps<E1>::value == 4, "four epilogue warps");
  static_assert(!epi_fp8<E0>::value && !epi_fp8<E1>::value && !E0::kPairedB && !E1::kPairedB,
                "plain bf16 operands");
};

// The tiles of pair `pr` (of np pairs).  Problem-0 tiles go round-robin:
// pair pr gets pr, pr + np, ...; the first a = n0 mod np pairs get one more
// than the rest.  A pair's capacity for problem-1 tiles is what fits under
// the makespan `target` (in k-blocks) beside its problem-0 tiles: cap_a for
// those first a pairs, cap_b >= cap_a for the others.  Problem-1 tiles are
// then dealt in rounds, consecutive ids to consecutive pairs (so the tiles
// running at the same time are neighbours in the raster and share operands
// in L2): rounds j < cap_a go to every pair, rounds cap_a <= j < cap_b only
// to pairs a .. np-1.  Ids from n1 on are not dealt.
struct PairTiles {
  int pr, np, n1;
  int nl;            // problem-0 tiles of this pair
  int ns;            // problem-1 tiles of this pair
  int a, cap_a;      // pairs with one more problem-0 tile; their capacity
  __device__ __forceinline__ int count() const { return nl + ns; }
  __device__ __forceinline__ int short_id(int j) const {
    return j < cap_a ? j * np + pr : cap_a * np + (j - cap_a) * (np - a) + (pr - a);
  }
};

__host__ __device__ __forceinline__ int grouped_cap(int target, int nl, int u0, int u1) {
  const int room = target - nl * u0;
  return room > 0 ? room / u1 : 0;
}

__device__ __forceinline__ PairTiles pair_tiles(int pr, int np, int n0, int n1, int u0, int u1, int target) {
  PairTiles t;
  t.pr = pr;
  t.np = np;
  t.n1 = n1;
  const int lo = n0 / np;
  t.a = n0 - lo * np;
  t.nl = pr < t.a ? lo + 1 : lo;
  t.cap_a = grouped_cap(target, lo + 1, u0, u1);
  const int cap_b = grouped_cap(target, lo, u0, u1);
  const int cap = pr < t.a ? t.cap_a : cap_b;
  if (t.a == 0) t.cap_a = cap_b;  // every pair alike: one capacity
  int ns = 0;
  while (ns < cap && t.short_id(ns) < n1) ++ns;
  t.ns = ns;
  return t;
}

template <int BN, int STAGES, class E0, class E1>
__global__ void __launch_bounds__(kThreads, 1) coda_gemm_grouped_kernel(const __grid_constant__ GroupedParams<E0, E1> p) {
  using S = GroupedSmem<E0, E1>;
  static_assert(BN == 256, "pair tiles are 256 x 256");
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
  uint64_t* ebars = drain + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(ebars + kEpiWarps * S::kBarsPerWarp);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int np = static_cast<int>(gridDim.x >> 1);
  const int pr = static_cast<int>(blockIdx.x >> 1);
  const int u0 = (p.K[0] + kBK - 1) / kBK;
  const int u1 = (p.K[1] + kBK - 1) / kBK;
  const PairTiles mine = pair_tiles(pr, np, p.ntiles[0], p.ntiles[1], u0, u1, p.target);
  const int nmine = mine.count();

  // tile i of this pair -> (problem, mb, nb)
  auto tile_at = [&](int i, int& prob, int& mb, int& nb) {
    int local;
    if (i < mine.nl) {
      prob = 0;
      local = pr + i * np;
    } else {
      prob = 1;
      local = mine.short_id(i - mine.nl);
    }
    TileSched sc;
    sc.n_mt = p.n_mt[prob];
    sc.n_nt = p.n_nt[prob];
    sc.group_m = p.group_m[prob];
    sc.ntiles = p.ntiles[prob];
    sc.map(local, mb, nb);
  };

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
    for (int i = 0; i < kEpiWarps * S::kBarsPerWarp; ++i) mbar_init(&ebars[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int q = 0; q < 2; ++q) {
      tma_prefetch_desc(&p.tmA[q]);
      tma_prefetch_desc(&p.tmB[q]);
    }
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
  // launched with programmatic serialisation: let the next kernel start its
  // prologue, and wait for the previous one before reading anything
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      const uint32_t full0 = mapa_shared(smem_u32(full), 0);
      for (int i = 0; ok && i < nmine; ++i) {
        int prob, mb, nb;
        tile_at(i, prob, mb, nb);
        const CUtensorMap* tA = &p.tmA[prob];
        const CUtensorMap* tB = &p.tmB[prob];
        const bool a_mn = p.a_mn[prob] != 0;
        const bool b_mn = p.b_mn[prob] != 0;
        const int nkb = prob == 0 ? u0 : u1;
        const int arow = mb * kTileM + static_cast<int>(rank) * kBM;
        const int bcol = nb * BN + static_cast<int>(rank) * kBCols;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, w)) {
            ok = false;
            break;
          }
          uint8_t* a = sA + stage * S::kABytes;
          uint8_t* b = sB + stage * S::kBBytes;
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * S::kStageBytes);
          const uint32_t fb = full0 + stage * 8;
          if (!a_mn) {
            tma_load_2d_pair(a, tA, fb, kb * kBK, arow);
          } else {
#pragma unroll
            for (int j = 0; j < kBM / 64; ++j) tma_load_2d_pair(a + j * (64 * kBK * 2), tA, fb, arow + j * 64, kb * kBK);
          }
          if (!b_mn) {
            tma_load_2d_pair(b, tB, fb, kb * kBK, bcol);
          } else {
#pragma unroll
            for (int j = 0; j < kBCols / 64; ++j)
              tma_load_2d_pair(b + j * (64 * kBK * 2), tB, fb, bcol + j * 64, kb * kBK);
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // the loads of a pair complete on rank 0's barriers: wait for the MMA's
      // release of each stage still in flight
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
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; ok && i < nmine; ++i) {
        int prob, mb, nb;
        tile_at(i, prob, mb, nb);
        const bool a_mn = p.a_mn[prob] != 0;
        const bool b_mn = p.b_mn[prob] != 0;
        const uint32_t idesc = idesc_bf16_f32(kTileM, BN, a_mn, b_mn);
        const int nkb = prob == 0 ? u0 : u1;
        const int acc = i & 1;
        const uint32_t aph = (i >> 1) & 1;
        if (!mbar_wait(&tempty[acc], aph ^ 1u, w)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * BN;
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
            const uint64_t ad = a_mn ? sdesc_sw128(a0 + kk * 16 * 128, 64 * kBK * 2, 1024)
                                     : sdesc_sw128(a0 + kk * 32, 16, 1024);
            const uint64_t bd = b_mn ? sdesc_sw128(b0 + kk * 16 * 128, 64 * kBK * 2, 1024)
                                     : sdesc_sw128(b0 + kk * 32, 16, 1024);
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
    uint8_t* wsmem = sEpi + ew * S::kPerWarp;
    uint64_t* wbars = ebars + ew * S::kBarsPerWarp;
    const uint32_t tempty0 = mapa_shared(smem_u32(tempty), 0);
    typename E0::State st0;
    typename E1::State st1;
    E0::init_state(st0);
    E1::init_state(st1);
    for (int i = 0; i < nmine; ++i) {
      int prob, mb, nb;
      tile_at(i, prob, mb, nb);
      const int acc = i & 1;
      const uint32_t aph = (i >> 1) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph, w))) break;
      tc_fence_after();
      if (prob == 1 && i == mine.nl && i > 0) {
        // the staging buffers change owners: each epilogue alternates its two
        // buffers by its own count, so the second one's first buffer may be
        // the one the first one's last store is still reading
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
      }
      TileCtx c;
      c.M = p.M[prob];
      c.N = p.N[prob];
      c.mb = mb;
      c.nb = nb;
      c.row0 = mb * kTileM + static_cast<int>(rank) * kBM + q * 32;
      c.taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * BN;
      c.lane = lane;
      c.wsmem = wsmem;
      c.wbars = wbars;
      c.has_next = false;  // a prefetch across tiles must stay within one problem
      c.nrow0 = 0;
      c.ncol0 = 0;
      if (i + 1 < nmine) {
        int nprob, nmb, nnb;
        tile_at(i + 1, nprob, nmb, nnb);
        if (nprob == prob) {
          c.has_next = true;
          c.nrow0 = nmb * kTileM + static_cast<int>(rank) * kBM + q * 32;
          c.ncol0 = nnb * BN;
        }
      }
      c.cend = BN;
      const bool ok = prob == 0 ? E0::template tile<BN>(p.ep0, c, st0, w) : E1::template tile<BN>(p.ep1, c, st1, w);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty0 + acc * 8);
      if (!ok) break;
    }
    E0::finish(p.ep0, st0, wbars, lane, p.wait_ns);
    E1::finish(p.ep1, st1, wbars, lane, p.wait_ns);
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
