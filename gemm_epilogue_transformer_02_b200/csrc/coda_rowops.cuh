// Row kernels of the CODA hot path (HBM- or latency-bound; no tensor cores):
// the light reduction that turns partial sums of squares into the RMSNorm row
// scale, the RMSNorm backward row reduction, the cross-entropy tile combine,
// and the separate add / RMSNorm kernels of the unfused comparison chain.
//
// Source: KuCoin news flash "CODA: new research optimizes transformer training
// with GEMM epilogue programming", section "CODA: the secret in the epilogue"
// (partial RMS from the first GEMM, combined by a light reduction kernel).
#pragma once

#include "coda_device.cuh"

namespace coda {

// r_i = 1 / sqrt(sum_t partial[t, i] / N + eps).  One thread per row; the
// partials of a column slot are contiguous over rows, so loads coalesce.
__global__ void rms_reduce_kernel(const float* __restrict__ partial, int M, int T, float inv_n, float eps,
                                  float* __restrict__ r) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= M) return;
  float s = 0.f;
  for (int t = 0; t < T; ++t) s += __ldg(partial + static_cast<size_t>(t) * M + i);
  r[i] = rsqrtf(s * inv_n + eps);
}

// RMSNorm backward row pass over a block of kBwdRows rows:
//   dr_i = sum_t pdr[t, i];  coef_i = -r_i^3 dr_i / N;
//   dh = gamma * d_hg + coef * h  (d_hg fp32, h bf16, dh bf16);  dgamma partial
//   over the block's rows.
// Each thread owns 8 consecutive columns and walks the rows, so every row
// access is a coalesced vector sweep; four rows at a time, their loads issued
// before any of them is used, so that enough bytes are in flight per SM to
// keep HBM busy.
constexpr int kBwdRows = 32;
constexpr int kBwdThreads = 256;
constexpr int kBwdUnroll = 4;

__global__ void __launch_bounds__(kBwdThreads) rms_reduce_bwd_kernel(
    const float* __restrict__ pdr, const float* __restrict__ r, const float* __restrict__ d_hg,
    const __nv_bfloat16* __restrict__ h, const __nv_bfloat16* __restrict__ gamma, __nv_bfloat16* __restrict__ dh,
    float* __restrict__ dgamma_part, int M, int T, int N) {
  __shared__ float coef[kBwdRows];
  const int r0 = blockIdx.x * kBwdRows;
  if (threadIdx.x < kBwdRows) {
    const int i = r0 + threadIdx.x;
    float c = 0.f;
    if (i < M) {
      float dr = 0.f;
      for (int t = 0; t < T; ++t) dr += pdr[static_cast<size_t>(t) * M + i];
      const float ri = r[i];
      c = -ri * ri * ri * dr / static_cast<float>(N);
    }
    coef[threadIdx.x] = c;
  }
  __syncthreads();
  const int nrows = min(kBwdRows, M - r0);
  for (int c0 = threadIdx.x * 8; c0 < N; c0 += kBwdThreads * 8) {
    const uint4 g4 = *reinterpret_cast<const uint4*>(gamma + c0);
    const uint32_t gw[4] = {g4.x, g4.y, g4.z, g4.w};
    float dg[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) dg[e] = 0.f;
    for (int rb = 0; rb < nrows; rb += kBwdUnroll) {
      float4 alo[kBwdUnroll], ahi[kBwdUnroll];
      uint4 hv[kBwdUnroll];
#pragma unroll
      for (int u = 0; u < kBwdUnroll; ++u) {
        if (rb + u < nrows) {
          const size_t o = static_cast<size_t>(r0 + rb + u) * N + c0;
          alo[u] = __ldcs(reinterpret_cast<const float4*>(d_hg + o));
          ahi[u] = __ldcs(reinterpret_cast<const float4*>(d_hg + o + 4));
          hv[u] = __ldcs(reinterpret_cast<const uint4*>(h + o));
        } else {
          alo[u] = ahi[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          hv[u] = make_uint4(0, 0, 0, 0);
        }
      }
#pragma unroll
      for (int u = 0; u < kBwdUnroll; ++u) {
        if (rb + u >= nrows) break;
        const size_t o = static_cast<size_t>(r0 + rb + u) * N + c0;
        const float av[8] = {alo[u].x, alo[u].y, alo[u].z, alo[u].w, ahi[u].x, ahi[u].y, ahi[u].z, ahi[u].w};
        const uint32_t hw[4] = {hv[u].x, hv[u].y, hv[u].z, hv[u].w};
        const float cf = coef[rb + u];
        uint32_t out[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a0 = av[2 * e], a1 = av[2 * e + 1];
          const float h0 = bf16lo(hw[e]), h1 = bf16hi(hw[e]);
          dg[2 * e] = fmaf(a0, h0, dg[2 * e]);
          dg[2 * e + 1] = fmaf(a1, h1, dg[2 * e + 1]);
          out[e] = pack_bf16x2(fmaf(bf16lo(gw[e]), a0, cf * h0), fmaf(bf16hi(gw[e]), a1, cf * h1));
        }
        // dh is read next by the dx and dW1 GEMMs: a plain store leaves it in L2
        *reinterpret_cast<uint4*>(dh + o) = make_uint4(out[0], out[1], out[2], out[3]);
      }
    }
    float* dst = dgamma_part + static_cast<size_t>(blockIdx.x) * N + c0;
    *reinterpret_cast<float4*>(dst) = make_float4(dg[0], dg[1], dg[2], dg[3]);
    *reinterpret_cast<float4*>(dst + 4) = make_float4(dg[4], dg[5], dg[6], dg[7]);
  }
}

// dgamma_j = sum over row blocks of the block partials, in a fixed order:
// a block of 256 threads takes 8 columns; thread (g, j) sums the partials of
// row blocks g, g + 32, g + 64, ... of column j, and the 32 group sums of a
// column are added in group order.  (N / 8 blocks: 256 for N = 2048, enough
// loads in flight for a latency-bound 2 MB read.)
constexpr int kDgCols = 8;
constexpr int kDgGroups = 32;

__global__ void __launch_bounds__(kDgCols * kDgGroups) dgamma_final_kernel(const float* __restrict__ part, int nblk,
                                                                         int N, float* __restrict__ dgamma) {
  __shared__ float red[kDgGroups][kDgCols];
  const int jl = threadIdx.x % kDgCols, grp = threadIdx.x / kDgCols;
  const int j = blockIdx.x * kDgCols + jl;
  float s = 0.f;
  if (j < N)
    for (int b = grp; b < nblk; b += kDgGroups) s += part[static_cast<size_t>(b) * N + j];
  red[grp][jl] = s;
  __syncthreads();
  if (grp == 0 && j < N) {
    float t = 0.f;
#pragma unroll
    for (int g = 0; g < kDgGroups; ++g) t += red[g][jl];
    dgamma[j] = t;
  }
}

// Cross-entropy combine: per row, merge the (max, sum-exp) pairs of all
// vocabulary tiles: m* = max_t m_t, s* = sum_t s_t exp(m_t - m*), lse = m* + log s*.
// Block = 8 warps x 32 rows: lane = row, warp = a slice of the tiles; the
// slices are merged in shared memory in a fixed order.
constexpr int kCombWarps = 8;

__global__ void __launch_bounds__(32 * kCombWarps) ce_combine_kernel(
    const float* __restrict__ ws_m, const float* __restrict__ ws_s, const float* __restrict__ zlab,
    const int64_t* __restrict__ labels, int M, int n_tiles, long long V, float* __restrict__ lse_out,
    float* __restrict__ loss_out) {
  constexpr float kL2E = 1.4426950408889634f;
  constexpr float kLN2 = 0.6931471805599453f;
  __shared__ float sm[kCombWarps][32];
  __shared__ float ss[kCombWarps][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int row = blockIdx.x * 32 + lane;
  const int per = (n_tiles + kCombWarps - 1) / kCombWarps;
  const int t0 = warp * per, t1 = min(n_tiles, t0 + per);
  float m = -INFINITY, s = 0.f;
  if (row < M) {
    for (int t = t0; t < t1; ++t) {
      const size_t o = static_cast<size_t>(t) * M + row;
      const float mt = ws_m[o], st = ws_s[o];
      const float mn = fmaxf(m, mt);
      s = s * exp2f((m - mn) * kL2E) + st * exp2f((mt - mn) * kL2E);
      m = mn;
    }
  }
  sm[warp][lane] = m;
  ss[warp][lane] = s;
  __syncthreads();
  if (warp == 0 && row < M) {
    float M_ = -INFINITY, S_ = 0.f;
    for (int k = 0; k < kCombWarps; ++k) {
      const float mt = sm[k][lane], st = ss[k][lane];
      if (mt == -INFINITY) continue;  // empty slice
      const float mn = fmaxf(M_, mt);
      S_ = S_ * exp2f((M_ - mn) * kL2E) + st * exp2f((mt - mn) * kL2E);
      M_ = mn;
    }
    const float lse = M_ + log2f(S_) * kLN2;
    const long long lab = labels[row];
    const float loss = (lab >= 0 && lab < V) ? lse - zlab[row] : __int_as_float(0x7fc00000);
    lse_out[row] = lse;
    loss_out[row] = loss;
  }
}

// mean = sum(loss) / M, one block, fixed summation order (deterministic).
__global__ void __launch_bounds__(1024) mean_kernel(const float* __restrict__ loss, int M, float* __restrict__ mean) {
  __shared__ float red[1024];
  float s = 0.f;
  for (int i = threadIdx.x; i < M; i += 1024) s += loss[i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 512; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *mean = red[0] / static_cast<float>(M);
}

// Data-parallel cross-entropy ("What CODA can do": the article is single-GPU;
// splitting the tokens over ranks is this library's).  A rank reports
// (sum of its tokens' losses, its token count); the caller sums the pairs over
// ranks (an all-reduce of 8 bytes); the global mean is sum / count and each
// token's loss weight in the backward is 1 / count.
__global__ void __launch_bounds__(1024) loss_stats_kernel(const float* __restrict__ loss, int M,
                                                          float* __restrict__ stats) {
  __shared__ float red[1024];
  float s = 0.f;
  for (int i = threadIdx.x; i < M; i += 1024) s += loss[i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 512; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    stats[0] = red[0];
    stats[1] = static_cast<float>(M);
  }
}

__global__ void ce_global_finish_kernel(const float* __restrict__ stats, int M, float* __restrict__ mean,
                                        float* __restrict__ d_loss) {
  const float sum = stats[0], count = stats[1];
  if (mean != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *mean = sum / count;
  if (d_loss != nullptr) {
    const float w = 1.0f / count;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < M; i += gridDim.x * blockDim.x) d_loss[i] = w;
  }
}

// Cross-entropy backward: exact label entries.  The chunked backward stores the
// gradient G in bf16; at each row's label entry G = d (p - 1) dominates its dW
// column, so the rounding dropped there (resid_i, recorded in fp32 by the
// gradient epilogue) is added back, chunk by chunk:
//   dH[i, :] += resid_i W[:, label_i]        (ce_label_dh_fix_kernel)
//   dW[:, v] += sum over rows i with label_i = v (in increasing i) of resid_i H[i, :]
//                                             (in the dW GEMM's epilogue)
// The rows are bucketed by the 256-column vocabulary tile of their label and
// sorted within a bucket by (label, row): a chunk's rows are then one run of
// the sorted array, a dW tile's label columns one ordered run within it, and
// every column sums its rows in a fixed order (deterministic, no
// floating-point atomics).
constexpr int kLabelTile = 256;  // vocabulary columns per bucket (the GEMM tile width)

// counts[b] = number of rows whose label lies in vocabulary tile b.
__global__ void ce_label_count_kernel(const int64_t* __restrict__ labels, int M, long long V, int* counts) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= M) return;
  const long long lab = labels[i];
  if (lab >= 0 && lab < V) atomicAdd(&counts[lab / kLabelTile], 1);
}

// Exclusive scan of counts[0, n) into start[0, n] (start[n] = total) and a copy
// of it into cursor[0, n).  One block of 1024 threads walks the array.
__global__ void __launch_bounds__(1024) ce_label_scan_kernel(const int* __restrict__ counts, int n, int* start,
                                                             int* cursor) {
  __shared__ int warp_sums[32];
  __shared__ int carry;
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int base = 0; base < n; base += 1024) {
    const int i = base + static_cast<int>(threadIdx.x);
    const int v = i < n ? counts[i] : 0;
    int x = v;  // inclusive scan within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_sums[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int w = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_sums[lane] = w;
    }
    __syncthreads();
    const int excl = carry + (wid > 0 ? warp_sums[wid - 1] : 0) + x - v;
    if (i < n) {
      start[i] = excl;
      cursor[i] = excl;
    }
    __syncthreads();
    if (threadIdx.x == 1023) carry = excl + v;
    __syncthreads();
  }
  if (threadIdx.x == 0) start[n] = carry;
}

// Drops (label, row) of every row with a label in [0, V) into its bucket, in
// arrival order.
__global__ void ce_label_fill_kernel(const int64_t* __restrict__ labels, int M, long long V, int* cursor,
                                     int2* __restrict__ unsorted) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= M) return;
  const long long lab = labels[i];
  if (lab < 0 || lab >= V) return;
  const int pos = atomicAdd(&cursor[lab / kLabelTile], 1);
  unsorted[pos] = make_int2(static_cast<int>(lab), i);
}

// Places every entry at its rank by (label, row) within its bucket (the keys
// are distinct, so the result does not depend on the arrival order).
__global__ void ce_label_sort_kernel(const int2* __restrict__ unsorted, const int* __restrict__ start, int n,
                                     int2* __restrict__ sorted) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= start[n]) return;
  const int2 me = unsorted[e];
  const int b = me.x / kLabelTile;
  const int s0 = start[b];
  const int s1 = start[b + 1];
  int rank = 0;
  for (int f = s0; f < s1; ++f) {
    const int2 o = unsorted[f];
    rank += (o.x < me.x || (o.x == me.x && o.y < me.y)) ? 1 : 0;
  }
  sorted[s0 + rank] = me;
}

// dH[i, :] += resid_i W[:, label_i] for the rows whose label lies in buckets
// [b0, b1) (one vocabulary chunk), run right after that chunk's GEMMs, which
// leave the chunk of W in L2.  One warp per (row, 256 columns of dH): each
// lane gathers its 8 elements of W's label column at once, then updates 8
// coalesced 128-byte segments of the dH row; every element is written by one
// thread once.
constexpr int kDhFixSpan = 8;  // 32-column slices per warp item

// dH[i, :] += resid_i W[:, label_i] for the rows whose labels lie in
// vocabulary buckets [b0, b1), as warp items (row, 256-column slice) dealt to
// warps `warp`, `warp + nwarps`, ...; every element receives one addend.
__device__ __forceinline__ void ce_label_dh_fix_range(const int2* __restrict__ entries, const int* __restrict__ start,
                                                      int b0, int b1, const float* __restrict__ resid,
                                                      const __nv_bfloat16* __restrict__ W, long long V, int K,
                                                      float* __restrict__ dH, long long warp, long long nwarps,
                                                      int lane) {
  const int first = start[b0];
  const long long n = start[b1] - first;
  const int groups = (K + 32 * kDhFixSpan - 1) / (32 * kDhFixSpan);
  for (long long w = warp; w < n * groups; w += nwarps) {
    const int2 en = entries[first + static_cast<int>(w / groups)];
    const int kbase = static_cast<int>(w % groups) * 32 * kDhFixSpan + lane;
    const float ri = resid[en.y];
    float wv[kDhFixSpan];
#pragma unroll
    for (int u = 0; u < kDhFixSpan; ++u) {
      const int k = kbase + 32 * u;
      wv[u] = k < K ? __bfloat162float(W[static_cast<size_t>(k) * V + en.x]) : 0.f;
    }
    float* d = dH + static_cast<size_t>(en.y) * K;
#pragma unroll
    for (int u = 0; u < kDhFixSpan; ++u) {
      const int k = kbase + 32 * u;
      if (k < K) d[k] += ri * wv[u];
    }
  }
}

__global__ void ce_label_dh_fix_kernel(const int2* __restrict__ entries, const int* __restrict__ start, int b0,
                                       int b1, const float* __restrict__ resid, const __nv_bfloat16* __restrict__ W,
                                       long long V, int K, float* __restrict__ dH) {
  ce_label_dh_fix_range(entries, start, b0, b1, resid, W, V, K, dH,
                        (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5,
                        (static_cast<long long>(gridDim.x) * blockDim.x) >> 5, threadIdx.x & 31);
}

// ------------------------------------------------------------- FP8 (e4m3)
// Per-tensor scaling for the FP8 block: s = amax / 448 (1 for an all-zero
// tensor) and codes = e4m3(t * (1 / s)), rounded to nearest even and
// saturated to +-448 (the KuCoin news flash "CODA: new research optimizes
// transformer training with GEMM epilogue programming" names FP8 in section
// "The lazy cost of training large models" only as the reason the non-GEMM
// share grows; the scaling scheme is this library's).

__device__ __forceinline__ float e4m3_scale(float amax) { return amax > 0.f ? amax / 448.0f : 1.0f; }

// amax |src| of n8 * 8 bf16 values, as fp32 bits by atomic max (non-negative
// floats order like their bits); *amax must be zero before the launch.
__global__ void __launch_bounds__(256) amax_bf16_kernel(const __nv_bfloat16* __restrict__ src, size_t n8,
                                                        unsigned* amax) {
  __shared__ unsigned wm[8];
  float m = 0.f;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 v = reinterpret_cast<const uint4*>(src)[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) m = fmaxf(m, fmaxf(fabsf(bf16lo(w[e])), fabsf(bf16hi(w[e]))));
  }
  const unsigned u = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = u;
  __syncthreads();
  if (threadIdx.x < 32) {
    const unsigned v = __reduce_max_sync(0xffffffffu, threadIdx.x < 8 ? wm[threadIdx.x] : 0u);
    if (threadIdx.x == 0 && v != 0u) atomicMax(amax, v);
  }
}

__global__ void fp8_scale_kernel(const float* amax, float* scale) { *scale = e4m3_scale(*amax); }

// codes of n8 * 8 bf16 values, row-major as the source.
__global__ void __launch_bounds__(256) quantize_e4m3_kernel(const __nv_bfloat16* __restrict__ src, size_t n8,
                                                            const float* __restrict__ amax, uint8_t* __restrict__ dst) {
  const float inv = 1.0f / e4m3_scale(*amax);
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 v = reinterpret_cast<const uint4*>(src)[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t q[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) q[e] = pack_e4m3x2(bf16lo(w[e]) * inv, bf16hi(w[e]) * inv);
    reinterpret_cast<uint2*>(dst)[i] = make_uint2(q[0] | (q[1] << 16), q[2] | (q[3] << 16));
  }
}

// MXFP8 codes of a row-major bf16 matrix [rows, cols] (cols % 128 == 0),
// blocked along the row: each thread takes one 32-element block, finds its
// largest magnitude, takes the smallest power-of-two scale 2^e that keeps it
// within the e4m3 range and writes the 32 codes of v * 2^-e (round to nearest
// even) and the E8M0 byte e + 127 into the A or the B scale layout (b_layout;
// B's bytes four times).  Scale bytes of the padding rows (up to a whole
// 128-row block for A, a whole 256-row tile for B) are set to 127 (scale 1).
__global__ void __launch_bounds__(256) mx_quantize_kernel(const __nv_bfloat16* __restrict__ src, int rows, int cols,
                                                          int b_layout, uint8_t* __restrict__ q,
                                                          uint8_t* __restrict__ sf) {
  const int nb = cols >> 5;
  const int nrb = (rows + 127) >> 7;
  const int ntl = (rows + 255) >> 8;
  const size_t total = static_cast<size_t>(b_layout ? ntl * 2 : nrb) * 128 * nb;
  for (size_t t = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int row = static_cast<int>(t / nb);
    const int j = static_cast<int>(t - static_cast<size_t>(row) * nb);
    int e = 0;
    if (row < rows) {
      const uint4* p = reinterpret_cast<const uint4*>(src + static_cast<size_t>(row) * cols + j * 32);
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = __ldg(p + u);
      float amax = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) amax = fmaxf(amax, fmaxf(fabsf(bf16lo(w[k])), fabsf(bf16hi(w[k]))));
      }
      e = mx_e4m3_exponent(amax);
      const float inv = exp2_neg(e);
      uint32_t out[8];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        const uint32_t c0 = pack_e4m3x2(bf16lo(w[0]) * inv, bf16hi(w[0]) * inv);
        const uint32_t c1 = pack_e4m3x2(bf16lo(w[1]) * inv, bf16hi(w[1]) * inv);
        const uint32_t c2 = pack_e4m3x2(bf16lo(w[2]) * inv, bf16hi(w[2]) * inv);
        const uint32_t c3 = pack_e4m3x2(bf16lo(w[3]) * inv, bf16hi(w[3]) * inv);
        out[2 * u] = c0 | (c1 << 16);
        out[2 * u + 1] = c2 | (c3 << 16);
      }
      uint4* d = reinterpret_cast<uint4*>(q + static_cast<size_t>(row) * cols + j * 32);
      d[0] = make_uint4(out[0], out[1], out[2], out[3]);
      d[1] = make_uint4(out[4], out[5], out[6], out[7]);
    }
    const uint8_t byte = static_cast<uint8_t>(e + 127);
    if (b_layout) {
      const size_t o = mx_sf_offset_b(row, j, ntl);
#pragma unroll
      for (int r = 0; r < 4; ++r) sf[o + r * 512] = byte;
    } else {
      sf[mx_sf_offset_a(row, j, nrb)] = byte;
    }
  }
}

// Transposing form: src [rows, cols] -> dst [cols, rows] (a weight stored
// K-major for the e4m3 mainloop), 64 x 64 tiles through shared memory.
// Needs cols % 8 == 0 and rows % 4 == 0.
constexpr int kQT = 64;
__global__ void __launch_bounds__(256) quantize_e4m3_t_kernel(const __nv_bfloat16* __restrict__ src, int rows,
                                                              int cols, const float* __restrict__ amax,
                                                              uint8_t* __restrict__ dst) {
  __shared__ uint8_t tile[kQT][kQT + 4];
  const float inv = 1.0f / e4m3_scale(*amax);
  const int r0 = blockIdx.y * kQT;
  const int c0 = blockIdx.x * kQT;
  for (int i = threadIdx.x; i < kQT * kQT / 8; i += blockDim.x) {
    const int rr = i >> 3;
    const int cc = (i & 7) * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r0 + rr < rows && c0 + cc < cols)
      v = *reinterpret_cast<const uint4*>(src + static_cast<size_t>(r0 + rr) * cols + c0 + cc);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t q = pack_e4m3x2(bf16lo(w[e]) * inv, bf16hi(w[e]) * inv);
      tile[rr][cc + 2 * e] = static_cast<uint8_t>(q & 0xffu);
      tile[rr][cc + 2 * e + 1] = static_cast<uint8_t>(q >> 8);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kQT * kQT / 4; i += blockDim.x) {
    const int cc = i >> 4;
    const int rr = (i & 15) * 4;
    if (c0 + cc < cols && r0 + rr < rows) {
      const uint32_t q = static_cast<uint32_t>(tile[rr][cc]) | (static_cast<uint32_t>(tile[rr + 1][cc]) << 8) |
                         (static_cast<uint32_t>(tile[rr + 2][cc]) << 16) |
                         (static_cast<uint32_t>(tile[rr + 3][cc]) << 24);
      *reinterpret_cast<uint32_t*>(dst + static_cast<size_t>(c0 + cc) * rows + r0 + rr) = q;
    }
  }
}

// ------------------------------------------------------ unfused comparison chain

// out = a + b (bf16, 8 elements per thread).
__global__ void add_bf16_kernel(const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b,
                                __nv_bfloat16* __restrict__ out, size_t n8) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 x = reinterpret_cast<const uint4*>(a)[i];
    const uint4 y = reinterpret_cast<const uint4*>(b)[i];
    const uint32_t xw[4] = {x.x, x.y, x.z, x.w}, yw[4] = {y.x, y.y, y.z, y.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] = pack_bf16x2(bf16lo(xw[e]) + bf16lo(yw[e]), bf16hi(xw[e]) + bf16hi(yw[e]));
    reinterpret_cast<uint4*>(out)[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// Standalone RMSNorm: y = gamma * h / sqrt(mean(h^2) + eps), one block per row.
constexpr int kNormThreads = 256;

__global__ void __launch_bounds__(kNormThreads) rmsnorm_kernel(const __nv_bfloat16* __restrict__ h,
                                                              const __nv_bfloat16* __restrict__ gamma, float eps,
                                                              __nv_bfloat16* __restrict__ y, float* __restrict__ r_out,
                                                              int N) {
  __shared__ float red[kNormThreads / 32];
  const size_t rowoff = static_cast<size_t>(blockIdx.x) * N;
  float s = 0.f;
  for (int c = threadIdx.x * 8; c < N; c += kNormThreads * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(h + rowoff + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a = bf16lo(w[e]), b = bf16hi(w[e]);
      s = fmaf(a, a, fmaf(b, b, s));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int k = 0; k < kNormThreads / 32; ++k) tot += red[k];
  const float rr = rsqrtf(tot / static_cast<float>(N) + eps);
  if (threadIdx.x == 0 && r_out != nullptr) r_out[blockIdx.x] = rr;
  for (int c = threadIdx.x * 8; c < N; c += kNormThreads * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(h + rowoff + c);
    const uint4 g = *reinterpret_cast<const uint4*>(gamma + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w}, gw[4] = {g.x, g.y, g.z, g.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      o[e] = pack_bf16x2(bf16lo(gw[e]) * bf16lo(w[e]) * rr, bf16hi(gw[e]) * bf16hi(w[e]) * rr);
    *reinterpret_cast<uint4*>(y + rowoff + c) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// The same with an e4m3 output for the unfused FP8 chain: y8 = e4m3(y / s_y)
// (s_y a device float), amax = max |y| (fp32 bits by atomic max; zeroed by
// the caller).  N % 8 == 0.
__global__ void __launch_bounds__(kNormThreads) rmsnorm_e4m3_kernel(
    const __nv_bfloat16* __restrict__ h, const __nv_bfloat16* __restrict__ gamma, float eps,
    const float* __restrict__ s_y, uint8_t* __restrict__ y8, float* __restrict__ r_out, unsigned* amax, int N) {
  __shared__ float red[kNormThreads / 32];
  __shared__ unsigned mx[kNormThreads / 32];
  const size_t rowoff = static_cast<size_t>(blockIdx.x) * N;
  float s = 0.f;
  for (int c = threadIdx.x * 8; c < N; c += kNormThreads * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(h + rowoff + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a = bf16lo(w[e]), b = bf16hi(w[e]);
      s = fmaf(a, a, fmaf(b, b, s));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int k = 0; k < kNormThreads / 32; ++k) tot += red[k];
  const float rr = rsqrtf(tot / static_cast<float>(N) + eps);
  if (threadIdx.x == 0 && r_out != nullptr) r_out[blockIdx.x] = rr;
  const float inv = 1.0f / __ldg(s_y);
  float m = 0.f;
  for (int c = threadIdx.x * 8; c < N; c += kNormThreads * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(h + rowoff + c);
    const uint4 g = *reinterpret_cast<const uint4*>(gamma + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w}, gw[4] = {g.x, g.y, g.z, g.w};
    uint32_t q[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float y0 = bf16lo(gw[e]) * bf16lo(w[e]) * rr;
      const float y1 = bf16hi(gw[e]) * bf16hi(w[e]) * rr;
      m = fmaxf(m, fmaxf(fabsf(y0), fabsf(y1)));
      q[e] = pack_e4m3x2(y0 * inv, y1 * inv);
    }
    *reinterpret_cast<uint2*>(y8 + rowoff + c) = make_uint2(q[0] | (q[1] << 16), q[2] | (q[3] << 16));
  }
  const unsigned u = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
  if ((threadIdx.x & 31) == 0) mx[threadIdx.x >> 5] = u;
  __syncthreads();
  if (threadIdx.x < 32) {
    const unsigned t = __reduce_max_sync(0xffffffffu, threadIdx.x < kNormThreads / 32 ? mx[threadIdx.x] : 0u);
    if (threadIdx.x == 0 && t != 0u) atomicMax(amax, t);
  }
}

// ------------------------------------------------------------ bounded-wait self test

// Waits on an mbarrier that nothing ever arrives on, with the given limit.
// The wait must give up, record a timeout in the status word and return.
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns, int* gave_up) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    WaitCtx w{&abort_flag, limit_ns};
    const bool ok = mbar_wait(&bar, 0, w);
    *gave_up = ok ? 0 : 1;
  }
}

}  // namespace coda
