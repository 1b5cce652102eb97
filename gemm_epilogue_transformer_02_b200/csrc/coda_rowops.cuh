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
// partials of a column tile are contiguous over rows, so loads coalesce.
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
// access is a coalesced vector sweep.
constexpr int kBwdRows = 32;
constexpr int kBwdThreads = 256;

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
    for (int rr = 0; rr < nrows; ++rr) {
      const size_t o = static_cast<size_t>(r0 + rr) * N + c0;
      const float4 a4lo = *reinterpret_cast<const float4*>(d_hg + o);
      const float4 a4hi = *reinterpret_cast<const float4*>(d_hg + o + 4);
      const uint4 h4 = *reinterpret_cast<const uint4*>(h + o);
      const float av[8] = {a4lo.x, a4lo.y, a4lo.z, a4lo.w, a4hi.x, a4hi.y, a4hi.z, a4hi.w};
      const uint32_t hw[4] = {h4.x, h4.y, h4.z, h4.w};
      const float cf = coef[rr];
      uint32_t out[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a0 = av[2 * e], a1 = av[2 * e + 1];
        const float h0 = bf16lo(hw[e]), h1 = bf16hi(hw[e]);
        dg[2 * e] = fmaf(a0, h0, dg[2 * e]);
        dg[2 * e + 1] = fmaf(a1, h1, dg[2 * e + 1]);
        out[e] = pack_bf16x2(fmaf(bf16lo(gw[e]), a0, cf * h0), fmaf(bf16hi(gw[e]), a1, cf * h1));
      }
      *reinterpret_cast<uint4*>(dh + o) = make_uint4(out[0], out[1], out[2], out[3]);
    }
    float* dst = dgamma_part + static_cast<size_t>(blockIdx.x) * N + c0;
    *reinterpret_cast<float4*>(dst) = make_float4(dg[0], dg[1], dg[2], dg[3]);
    *reinterpret_cast<float4*>(dst + 4) = make_float4(dg[4], dg[5], dg[6], dg[7]);
  }
}

// dgamma_j = sum over row blocks (fixed order) of the block partials.
__global__ void dgamma_final_kernel(const float* __restrict__ part, int nblk, int N, float* __restrict__ dgamma) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= N) return;
  float s = 0.f;
  for (int b = 0; b < nblk; ++b) s += part[static_cast<size_t>(b) * N + j];
  dgamma[j] = s;
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

// Cross-entropy backward: exact label entries.  The chunked backward stores the
// gradient G in bf16; at each row's label entry G = d (p - 1) dominates its dW
// column, so the rounding dropped there (resid_i, recorded in fp32 by the
// gradient epilogue) is added back:
//   dH[i, :] += resid_i W[:, label_i]
//   dW[:, v] += sum over rows i with label_i = v (in increasing i) of resid_i H[i, :]
// Block i handles row i; the first row carrying a label owns that dW column,
// so every column is updated by one block in a fixed order (no atomics).
constexpr int kFixThreads = 256;
constexpr int kFixCols = 8;  // columns of dW per thread per pass

__global__ void __launch_bounds__(kFixThreads) ce_bwd_label_fix_kernel(
    const int64_t* __restrict__ labels, const float* __restrict__ resid, const __nv_bfloat16* __restrict__ H,
    const __nv_bfloat16* __restrict__ W, float* __restrict__ dH, float* __restrict__ dW, int M, int K,
    long long V) {
  __shared__ int rows[kFixThreads];
  __shared__ int warp_count[kFixThreads / 32];
  __shared__ int nrows;
  const int i = blockIdx.x;
  const long long lab = labels[i];
  if (lab < 0 || lab >= V) return;  // such a row has no label entry (and no residual)
  const float ri = resid[i];
  for (int k = threadIdx.x; k < K; k += kFixThreads)
    dH[static_cast<size_t>(i) * K + k] += ri * __bfloat162float(W[static_cast<size_t>(k) * V + lab]);
  int earlier = 0;
  for (int j = threadIdx.x; j < i; j += kFixThreads) earlier |= (labels[j] == lab);
  if (__syncthreads_or(earlier)) return;  // an earlier row owns this column
  // This block owns column `lab`.  Usually no later row repeats the label:
  // then the column gets resid_i H[i, :] alone.
  int later = 0;
  for (int j = i + 1 + static_cast<int>(threadIdx.x); j < M; j += kFixThreads) later |= (labels[j] == lab);
  if (!__syncthreads_or(later)) {
    for (int k = threadIdx.x; k < K; k += kFixThreads)
      dW[static_cast<size_t>(k) * V + lab] += ri * __bfloat162float(H[static_cast<size_t>(i) * K + k]);
    return;
  }
  // Otherwise add the residuals of rows j >= i carrying the same label, in
  // increasing j, kFixThreads * kFixCols columns per pass.
  for (int kbase = 0; kbase < K; kbase += kFixThreads * kFixCols) {
    float acc[kFixCols];
#pragma unroll
    for (int q = 0; q < kFixCols; ++q) acc[q] = 0.f;
    for (int j0 = i; j0 < M; j0 += kFixThreads) {
      const int j = j0 + threadIdx.x;
      const bool match = j < M && labels[j] == lab;
      const unsigned ballot = __ballot_sync(0xffffffffu, match);
      if ((threadIdx.x & 31) == 0) warp_count[threadIdx.x >> 5] = __popc(ballot);
      __syncthreads();
      int base = 0;
      for (int w = 0; w < (threadIdx.x >> 5); ++w) base += warp_count[w];
      if (match) rows[base + __popc(ballot & ((1u << (threadIdx.x & 31)) - 1u))] = j;
      if (threadIdx.x == 0) {
        int t = 0;
        for (int w = 0; w < kFixThreads / 32; ++w) t += warp_count[w];
        nrows = t;
      }
      __syncthreads();
      for (int q = 0; q < nrows; ++q) {
        const int jr = rows[q];
        const float rj = resid[jr];
#pragma unroll
        for (int s2 = 0; s2 < kFixCols; ++s2) {
          const int k = kbase + s2 * kFixThreads + threadIdx.x;
          if (k < K) acc[s2] += rj * __bfloat162float(H[static_cast<size_t>(jr) * K + k]);
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int s2 = 0; s2 < kFixCols; ++s2) {
      const int k = kbase + s2 * kFixThreads + threadIdx.x;
      if (k < K) dW[static_cast<size_t>(k) * V + lab] += acc[s2];
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
