/*
 * coda.h - C ABI of the CODA GEMM + epilogue hot path for NVIDIA B200 (sm_100a).
 *
 * Source of the operations: KuCoin news flash "CODA: new research optimizes
 * transformer training with GEMM epilogue programming".
 *   - Section "CODA: the secret in the epilogue": the GEMM-RMSNorm-GEMM
 *     pattern (matmul, residual add, RMS normalisation, second matmul).  The
 *     RMSNorm row scale r is one scalar per row, so it commutes with the
 *     second matmul and is applied in that GEMM's epilogue; the first GEMM's
 *     epilogue only emits a partial RMS, which a light reduction kernel
 *     combines; SwiGLU, cross-entropy and the backward pass get the same
 *     treatment, and a block-local forward epilogue gives a block-local
 *     backward.
 *   - Section "Five kinds of building blocks": elementwise transforms
 *     (residual add, activation), vector loads (RMSNorm weight broadcast),
 *     matrix-block loads/stores (saving activations for the backward), chunk
 *     reductions (local RMS, chunk log-sum-exp) and stateful transforms
 *     (running max and sum-exp of online normalisation).
 *
 * Conventions (all calls):
 *   - Every tensor pointer is a DEVICE pointer owned by the caller (the one
 *     exception, coda_rmsnorm_block_host, says which of its pointers are host
 *     memory); the library never allocates device memory for a call, frees
 *     or keeps a pointer after the call returns.  Scratch space is passed in
 *     by the caller, sized by the *_workspace_size queries.  What the library
 *     keeps for the life of the process: per device, the kernel attributes it
 *     has set, the device status word, the static scratch array of
 *     coda_rms_reduce_bwd_noalloc, and the two streams and six events of
 *     coda_rmsnorm_block_host (created on its first call).
 *   - Tensors are dense row-major.  Weights are stored [in, out]; activations
 *     [tokens, features].  bf16 tensors are passed as uint16_t bit patterns
 *     (IEEE bfloat16); float tensors are fp32; labels are int64.
 *   - Every tensor base pointer must be 16-byte aligned.  M (tokens) may be any
 *     value >= 0 (M == 0 is a no-op); feature sizes N, K, F, V must be > 0 and
 *     multiples of 8 (the tensor-memory-access copies need 16-byte rows), of
 *     16 where an e4m3 (1-byte) tensor has that row length.
 *   - Outputs must not alias inputs unless a call says otherwise.
 *   - Each call enqueues its kernels on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream) and returns without synchronising.  Calls are
 *     reentrant and keep no state between calls beyond what is listed above.
 *     The GEMM kernels use programmatic dependent launch: one may start its
 *     prologue while the previous GEMM on the stream finishes, but reads
 *     nothing before that kernel has completed, so stream order holds as
 *     for any launch.
 *   - Arithmetic: bf16 inputs (e4m3 for the FP8 calls), fp32 accumulation in
 *     tensor memory, fp32 epilogue math, bf16 outputs rounded to nearest-even.
 *   - Return value: CODA_OK, or an error.  Argument errors (NULL, SHAPE,
 *     ALIGN, WORKSPACE) are detected on the host before any CUDA call and
 *     nothing is launched.  CODA_ERR_DEVICE: the current device is not
 *     compute capability 10.0 (B200).  CODA_ERR_LAUNCH: a CUDA runtime call
 *     failed (the CUDA error is left for the caller to query).  Kernels never
 *     trap: a wait that exceeds its time limit records CODA_ERR_DEVICE_TIMEOUT
 *     in the device status word, which coda_poll_status() reports.
 */
#ifndef CODA_H_
#define CODA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum coda_status_t {
  CODA_OK = 0,
  CODA_ERR_NULL = 1,           /* a required pointer is NULL */
  CODA_ERR_SHAPE = 2,          /* a size is negative, zero where it must not be, or not a multiple of 8 */
  CODA_ERR_ALIGN = 3,          /* a pointer is not 16-byte aligned */
  CODA_ERR_WORKSPACE = 4,      /* workspace missing or smaller than *_workspace_size */
  CODA_ERR_DEVICE = 5,         /* no device, or not sm_100 */
  CODA_ERR_LAUNCH = 6,         /* a CUDA runtime call failed */
  CODA_ERR_DEVICE_TIMEOUT = 7, /* a kernel gave up on a bounded wait (from coda_poll_status) */
  CODA_ERR_INTERNAL = 8        /* unexpected internal failure (e.g. tensor-map encoding) */
} coda_status_t;

/* Human-readable name of a status code (static string, never NULL). */
const char* coda_status_string(coda_status_t s);

/* Library ABI version (increments on any signature change). */
int coda_version(void);

/* Columns summed into one entry of the partial-sum layouts (partial, pdr):
 * 128, one half of a 256-column GEMM tile (the halves of a tile may be
 * computed by different CTA pairs when a GEMM's last wave is split). */
int64_t coda_partial_tile_width(void);

/* Number of column slots T = ceil(N / coda_partial_tile_width()) for a hidden
 * size N; partial and pdr arrays are [T, M] fp32 (slot-major: entry (t, i) at
 * index t * M + i).  Returns -1 if N <= 0. */
int64_t coda_partial_cols(int64_t N);

/* Sets the time limit of every bounded device wait (nanoseconds, > 0;
 * default 1e9).  Affects later launches only.  Returns CODA_ERR_SHAPE if <= 0. */
coda_status_t coda_set_wait_limit_ns(int64_t ns);

/* Synchronises `stream`, then reads and clears the device status word.
 * Returns CODA_ERR_DEVICE_TIMEOUT if any kernel recorded a timeout since the
 * last poll, CODA_ERR_LAUNCH if the stream reported a CUDA error, else CODA_OK. */
coda_status_t coda_poll_status(void* stream);

/* ---------------------------------------------------------------- forward */

/* First GEMM of the block with the residual + partial-RMS epilogue
 * (section "CODA: the secret in the epilogue": the first GEMM only computes a
 * partial RMS while its output is on chip).
 *   acc = x W (fp32);  h = acc + res (res may be NULL: h = acc);
 *   h_out  = bf16(h)                     [M, N]  (NULL: not stored)
 *   hg_out = bf16(gamma * h)             [M, N]  (NULL: not stored; needs gamma)
 *   partial[t, i] = sum_{j in slot t} h_ij^2 (fp32, from the unrounded h) [T, M] (NULL: not stored;
 *                   slot t = columns [128 t, 128 t + 128))
 * x [M, K] bf16, W [K, N] bf16, res [M, N] bf16, gamma [N] bf16.
 * At least one output must be non-NULL.  Also used as the down projection of
 * the SwiGLU chain (x = act, res = h, partials for the next layer's norm). */
coda_status_t coda_gemm_res_partialrms(const uint16_t* x, const uint16_t* W, const uint16_t* res,
                                       const uint16_t* gamma, uint16_t* h_out, uint16_t* hg_out, float* partial,
                                       int64_t M, int64_t N, int64_t K, void* stream);

/* The light reduction: r_i = 1 / sqrt(sum_t partial[t, i] / N + eps).
 * partial [T, M] fp32 with T = coda_partial_cols(N); r_out [M] fp32; eps >= 0. */
coda_status_t coda_rms_reduce(const float* partial, int64_t M, int64_t T, int64_t N, float eps, float* r_out,
                              void* stream);

/* Second GEMM with the RMSNorm row scale in its epilogue (r commutes with the
 * matmul): out = bf16(r_i * (A W)_ij); r == NULL gives a plain bf16 GEMM.
 * A [M, K] bf16 (hg of the first GEMM), W [K, N] bf16, r [M] fp32, out [M, N] bf16. */
coda_status_t coda_gemm_rowscale(const uint16_t* A, const uint16_t* W, const float* r, uint16_t* out, int64_t M,
                                 int64_t N, int64_t K, void* stream);

/* Second GEMM with the light reduction folded into its epilogue: each output
 * row's scale r_i = 1 / sqrt(sum_t partial[t, i] / N_norm + eps) is formed by
 * the epilogue from the first GEMM's partials (same summation order as
 * coda_rms_reduce, so the same r), then out = bf16(r_i * (A W)_ij).  r_out
 * [M] fp32 (may be NULL) receives r for the backward.  One launch instead of
 * two for the block's second half.  partial [T, M] fp32, A [M, K], W [K, N],
 * out [M, N] bf16; N_norm is the hidden size the partials were taken over.
 * Launched with programmatic stream serialisation: its CTAs may run their
 * prologue while the preceding kernel on the stream (coda_gemm_res_partialrms
 * lets them) still finishes, but read nothing before that kernel has
 * completed, so the stream order holds as for any launch.  The same holds
 * for coda_gemm_rowscale_partial_fp8 after coda_gemm_res_partialrms_fp8. */
coda_status_t coda_gemm_rowscale_partial(const uint16_t* A, const uint16_t* W, const float* partial, int64_t T,
                                         int64_t N_norm, float eps, float* r_out, uint16_t* out, int64_t M,
                                         int64_t N, int64_t K, void* stream);

/* Bytes of workspace coda_rmsnorm_block needs (one int per 256-row block). */
size_t coda_rmsnorm_block_workspace_size(int64_t M);

/* The whole GEMM-RMSNorm-GEMM block in one persistent launch: the work of
 * coda_gemm_res_partialrms (h, hg, partial) followed by that of
 * coda_gemm_rowscale_partial (out, r), with the same results.  Both GEMMs run
 * on the same CTA pairs: every pair first computes its share of first-GEMM
 * tiles, then second-GEMM tiles, each of which starts once all first-GEMM
 * tiles of its 256-row block have published their outputs (a counter per row
 * block in the workspace, zeroed by this call with a memset on `stream`).  The
 * second GEMM's tiles thereby fill the SMs the first GEMM's last wave leaves
 * idle.  The kernel needs all of its clusters resident at once (its grid is
 * the occupancy limit); kernels running concurrently on other streams that
 * keep part of it from becoming resident make its bounded waits expire
 * (CODA_ERR_DEVICE_TIMEOUT from coda_poll_status), so run it alone.
 * x [M, K], res [M, N] (or NULL), W1 [K, N], W2 [N, N2], gamma [N] bf16;
 * h_out, hg_out [M, N] bf16; partial_out [T, M] fp32 (T = coda_partial_cols(N));
 * r_out [M] fp32 (or NULL); out [M, N2] bf16. */
coda_status_t coda_rmsnorm_block(const uint16_t* x, const uint16_t* res, const uint16_t* W1, const uint16_t* W2,
                                 const uint16_t* gamma, float eps, uint16_t* h_out, uint16_t* hg_out,
                                 float* partial_out, float* r_out, uint16_t* out, void* ws, size_t ws_bytes,
                                 int64_t M, int64_t K, int64_t N, int64_t N2, void* stream);

/* Gate/up GEMM with SwiGLU in its epilogue (section "CODA: the secret in the
 * epilogue" lists SwiGLU among the re-parameterised operations):
 *   g = r_i (A W_gu[:, :F])_ij,  u = r_i (A W_gu[:, F:])_ij,  act = bf16(silu(g) * u)
 * with silu(g) = g / (1 + exp(-g)).  The [M, 2F] gate/up product never reaches
 * memory unless gateup_save is given (then bf16 g in columns [0, F) and u in
 * [F, 2F) of gateup_save [M, 2F], for the backward).
 * A [M, K] bf16, W_gu [K, 2F] bf16, r [M] fp32 or NULL (scale 1), act_out [M, F] bf16. */
coda_status_t coda_gemm_swiglu(const uint16_t* A, const uint16_t* W_gu, const float* r, uint16_t* act_out,
                               uint16_t* gateup_save, int64_t M, int64_t F, int64_t K, void* stream);

/* QKV projection with RoPE in its epilogue (section "CODA: the secret in the
 * epilogue" lists RoPE, rotary position encoding, among the re-parameterised
 * operations; section "Five kinds of building blocks": an elementwise
 * transform).  acc = x W_qkv (fp32); for every head of head_dim columns below
 * rope_cols (the q and k heads), columns i and i + head_dim/2 of the head are
 * rotated by the angle positions[m] * theta^(-2 i / head_dim):
 *   (a, b) -> (a cos - b sin, b cos + a sin);
 * columns from rope_cols on (v) are stored unrotated; out = bf16.
 * x [M, K] bf16, W_qkv [K, N] bf16 (q heads, then k heads, then v heads),
 * positions [M] int32 (any value, negative included), out [M, N] bf16;
 * head_dim 64 or 128, N and rope_cols multiples of head_dim, theta > 1
 * (LLaMA-3: 500000).  Each angle is reduced to a fraction of a turn exactly
 * (the position times the frequency in 2^-64 turn, in 64-bit integers) before
 * the fp32 sine and cosine, so long positions lose no accuracy. */
coda_status_t coda_gemm_qkv_rope(const uint16_t* x, const uint16_t* W_qkv, const int32_t* positions, uint16_t* out,
                                 int64_t M, int64_t N, int64_t K, int64_t head_dim, int64_t rope_cols, float theta,
                                 void* stream);

/* SwiGLU backward, block-local in the down projection's dA GEMM (section "CODA:
 * the secret in the epilogue": the backward of a block-local epilogue is
 * block-local too).  The GEMM forms d_act = d_out W_down^T tile by tile; its
 * epilogue reads the saved gate g and up u of the same tile (gateup, as saved
 * by coda_gemm_swiglu) and writes
 *   d_gateup[:, j]     = bf16(d_act_j * u_j * silu'(g_j))   (gate half)
 *   d_gateup[:, F + j] = bf16(d_act_j * silu(g_j))           (up half)
 * with silu'(g) = s (1 + g (1 - s)), s = 1 / (1 + exp(-g)); d_act is not
 * stored.  d_out [M, N] bf16 (gradient of the down projection's output),
 * W_down [F, N] bf16, gateup and d_gateup_out [M, 2F] bf16.  The rest of the
 * MLP backward are plain GEMMs: coda_gemm_res_partialrms_bwd(d_gateup, y, W_gu)
 * gives d_y and dW_gu; with x = act it gives dW_down. */
coda_status_t coda_gemm_swiglu_bwd(const uint16_t* d_out, const uint16_t* W_down, const uint16_t* gateup,
                                   uint16_t* d_gateup_out, int64_t M, int64_t F, int64_t N, void* stream);

/* Bytes of workspace coda_lmhead_ce needs for M tokens and vocabulary V. */
size_t coda_lmhead_ce_workspace_size(int64_t M, int64_t V);

/* LM-head cross-entropy with a block log-sum-exp epilogue (section "Five kinds
 * of building blocks": chunk log-sum-exp and the running max / sum-exp of
 * online normalisation).  Logits z = r_i (H W)_ij (fp32, never stored; r NULL
 * means scale 1).  Per token lse_i = log sum_j exp(z_ij), loss_i = lse_i -
 * z_{i,label_i} (natural log); mean = sum_i loss_i / M.  A label outside
 * [0, V) gives a NaN loss for that token (no device trap).
 * H [M, K] bf16, W [K, V] bf16, labels [M] int64, loss_out/lse_out [M] fp32,
 * mean_out [1] fp32 (may be NULL), ws >= coda_lmhead_ce_workspace_size(M, V). */
coda_status_t coda_lmhead_ce(const uint16_t* H, const uint16_t* W, const int64_t* labels, const float* r,
                             float* loss_out, float* lse_out, float* mean_out, void* ws, size_t ws_bytes,
                             int64_t M, int64_t V, int64_t K, void* stream);

/* Bytes of workspace coda_lmhead_ce_bwd needs: one bf16 gradient chunk of
 * M x min(V, 8192), M fp32 residuals, and the rows bucketed by label (three
 * int arrays of ceil(V / 256) entries and two of M (label, row) pairs). */
size_t coda_lmhead_ce_bwd_workspace_size(int64_t M, int64_t V);

/* Backward of coda_lmhead_ce, block-local (section "CODA: the secret in the
 * epilogue": the backward inherits the block-local structure).  For the loss
 * L = sum_i d_i loss_i (d = d_loss, or 1/M for every token when d_loss is
 * NULL: the mean), with the forward's saved lse:
 *   G_ij = d_i (exp(z_ij - lse_i) - [j == label_i]),  z = r_i (H W)_ij
 *   dH_out = G W^T  [M, K] fp32;   dW_out = H^T G  [K, V] fp32.
 * The vocabulary is processed in chunks of 8192 columns: a GEMM recomputes the
 * chunk's logits and its epilogue writes G_chunk (bf16, in the workspace;
 * the logits are never stored), then dH += G_chunk W_chunk^T (the first
 * chunk stores, later chunks add in fp32 through TMA reduce-adds, in chunk
 * order) and dW_chunk = H^T G_chunk run as one grouped launch.  The label entry d_i (p - 1) dominates its dW
 * column, so the part of it that bf16 drops is kept in fp32 and added back:
 * into dW in the dW GEMM's epilogue (rows bucketed by label beforehand; each
 * dW column sums its rows in increasing row order, so the result is
 * deterministic), into dH by the next chunk's gradient GEMM before its first
 * tile (by a small kernel after the last chunk).  A label outside [0, V) contributes no onehot term.  H [M, K] bf16,
 * W [K, V] bf16, labels [M] int64, lse [M] fp32, d_loss and r [M] fp32 or NULL,
 * ws >= coda_lmhead_ce_bwd_workspace_size(M, V). */
coda_status_t coda_lmhead_ce_bwd(const uint16_t* H, const uint16_t* W, const int64_t* labels, const float* lse,
                                 const float* d_loss, const float* r, float* dH_out, float* dW_out, void* ws,
                                 size_t ws_bytes, int64_t M, int64_t V, int64_t K, void* stream);

/* Data-parallel cross-entropy (tokens split over ranks; the article is
 * single-GPU, section "What CODA can do").  stats_out[0] = sum of loss[0..M),
 * stats_out[1] = M (fp32; one block, fixed order: deterministic; a NaN loss
 * makes the sum NaN).  The caller sums stats over ranks (an all-reduce of 8
 * bytes).  loss [M] fp32, stats_out [2] fp32, device.  0 < M < 2^24. */
coda_status_t coda_loss_stats(const float* loss, int64_t M, float* stats_out, void* stream);

/* From the rank-summed stats: mean_out[0] = stats[0] / stats[1] (the mean
 * over every rank's tokens) and d_loss_out[i] = 1 / stats[1] for i < M, the
 * per-token weight that coda_lmhead_ce_bwd takes as d_loss so that dW is the
 * gradient of the global mean (to be summed over ranks).  Either output may
 * be NULL, not both.  stats [2], mean_out [1], d_loss_out [M]: device fp32. */
coda_status_t coda_ce_global_finish(const float* stats, int64_t M, float* mean_out, float* d_loss_out,
                                    void* stream);

/* ---------------------------------------------------------------- backward *//* ---------------------------------------------------------------- backward */

/* Bytes of workspace coda_gemm_rowscale_bwd needs (holds y = r * hg, bf16 [M, N]). */
size_t coda_gemm_rowscale_bwd_workspace_size(int64_t M, int64_t N);

/* Backward of out = r * (hg W2) in block-local form.
 *   P = dOut W2^T (fp32, on chip);  d_hg_out = r * P (fp32)           [M, N]
 *   y = bf16(r * hg) (workspace);  pdr[t, i] = sum_{j in slot t} hg_ij P_ij   [T, M] fp32
 *   dW2_out = y^T dOut (fp32)                                          [N, N2]
 * dOut [M, N2] bf16, hg [M, N] bf16, W2 [N, N2] bf16, r [M] fp32.
 * d_hg and pdr feed coda_rms_reduce_bwd.  When the tiles of a GEMM end in a
 * partial wave on at most half of the CTA pairs and its K is 4096 or more,
 * that wave is split by k-blocks: the call first zeroes the part of d_hg and
 * pdr (or dW2) those tiles cover, and two units add their halves into it
 * (in fp32; the same bits from call to call). */
coda_status_t coda_gemm_rowscale_bwd(const uint16_t* dOut, const uint16_t* hg, const uint16_t* W2, const float* r,
                                     float* d_hg_out, float* dW2_out, float* pdr_out, void* ws, size_t ws_bytes,
                                     int64_t M, int64_t N, int64_t N2, void* stream);

/* Bytes of workspace coda_rms_reduce_bwd needs (per-row-block dgamma partials). */
size_t coda_rms_reduce_bwd_workspace_size(int64_t M, int64_t N);

/* RMSNorm backward row reduction:
 *   dr_i = sum_t pdr[t, i];  coef_i = -r_i^3 dr_i / N;
 *   dh_out = bf16(gamma * d_hg + coef_i * h)   [M, N]  (this is also dres)
 *   dgamma_out_j = sum_i d_hg_ij h_ij           [N] fp32 (fixed summation order)
 * pdr [T, M], r [M] fp32; d_hg [M, N] fp32; h [M, N] bf16; gamma [N] bf16.
 * d_hg is kept in fp32 so that dh is rounded to bf16 only once. */
coda_status_t coda_rms_reduce_bwd(const float* pdr, const float* r, const float* d_hg, const uint16_t* h,
                                  const uint16_t* gamma, uint16_t* dh_out, float* dgamma_out, void* ws,
                                  size_t ws_bytes, int64_t M, int64_t T, int64_t N, void* stream);

/* Same computation as coda_rms_reduce_bwd, for callers that cannot allocate
 * device memory at call time (a process whose device-memory budget is fixed
 * at start-up, or a framework that owns all device memory in its own pool and
 * cannot hand out a workspace).  It takes no workspace and allocates nothing:
 * the dgamma partials live in one static device array of 2^20 floats (4 MiB)
 * inside the library, held on every GPU that loads the library until the
 * process exits.  Limit: ceil(M / 32) * N <= 2^20 (for example M = 8192 with
 * N up to 4096); larger sizes return CODA_ERR_WORKSPACE and launch nothing.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * All calls on a device share the array: calls whose kernels overlap on the
 * GPU (other streams or threads) race and must be ordered by the caller.  The
 * array keeps the last call's contents; nothing in it needs to start at zero.
 * This entry point is a deployment convenience with no counterpart in the
 * CODA article. */
coda_status_t coda_rms_reduce_bwd_noalloc(const float* pdr, const float* r, const float* d_hg, const uint16_t* h,
                                          const uint16_t* gamma, uint16_t* dh_out, float* dgamma_out, int64_t M,
                                          int64_t T, int64_t N, void* stream);

/* Backward of h = x W1 + res: dx_out = bf16(dh W1^T) [M, K], dW1_out = x^T dh
 * (fp32) [K, N]; dres equals dh.  dh [M, N] bf16, x [M, K] bf16, W1 [K, N] bf16.
 * Either output may be NULL (not computed).  With both requested and M >= N
 * the two GEMMs share one persistent launch (the dW1 tiles first, the dx
 * tiles filling each CTA pair up to a common makespan); otherwise two, and
 * the dW1 GEMM may split its last partial wave by k-blocks as
 * coda_gemm_rowscale_bwd does (zeroing, then adding into, part of dW1_out). */
coda_status_t coda_gemm_res_partialrms_bwd(const uint16_t* dh, const uint16_t* x, const uint16_t* W1,
                                           uint16_t* dx_out, float* dW1_out, int64_t M, int64_t N, int64_t K,
                                           void* stream);

/* ------------------------------------------------- unfused comparison chain */

/* out = bf16(a + b), n elements (n a multiple of 8); the separate residual add
 * of the unfused GEMM -> add -> RMSNorm -> GEMM chain. */
coda_status_t coda_unfused_add(const uint16_t* a, const uint16_t* b, uint16_t* out, int64_t n, void* stream);

/* Standalone RMSNorm of the unfused chain: y = bf16(gamma * h / sqrt(mean_j h_ij^2 + eps)),
 * r_out [M] fp32 (may be NULL).  h, y [M, N] bf16; gamma [N] bf16. */
coda_status_t coda_unfused_rmsnorm(const uint16_t* h, const uint16_t* gamma, float eps, uint16_t* y_out,
                                   float* r_out, int64_t M, int64_t N, void* stream);

/* The block with host-resident activations: x [M, K] and res [M, N] (or
 * NULL) are read from host memory and out [M, N2] written to host memory;
 * W1, W2 and gamma are device pointers (resident weights).  The rows go
 * through in chunks of chunk_rows (a multiple of 256): while chunk i runs the
 * two GEMMs on `stream`, chunk i + 1 is copied in and chunk i - 1 copied out
 * on two streams of the library's own, so the copies overlap each other and
 * the compute.  Host buffers should be pinned (page-locked) for the copies
 * to overlap.  h, hg, partial and r stay in the workspace (two chunk slots,
 * coda_rmsnorm_block_host_workspace_size bytes).  On return the work is
 * queued; out_host is complete once `stream` is synchronised.  Results are
 * bitwise those of coda_gemm_res_partialrms + coda_gemm_rowscale_partial on
 * the whole batch.  Calls made at the same time from several host threads
 * on one device take turns while they enqueue (they share the library's two
 * copy streams and their events); their GPU work still overlaps.  On an error
 * part-way, `stream` still waits for the copies already queued. */
size_t coda_rmsnorm_block_host_workspace_size(int64_t K, int64_t N, int64_t N2, int64_t chunk_rows);
coda_status_t coda_rmsnorm_block_host(const uint16_t* x_host, const uint16_t* res_host, const uint16_t* W1,
                                      const uint16_t* W2, const uint16_t* gamma, float eps, uint16_t* out_host,
                                      void* ws, size_t ws_bytes, int64_t M, int64_t K, int64_t N, int64_t N2,
                                      int64_t chunk_rows, void* stream);

/* ------------------------------------------------------------ FP8 (e4m3)
 *
 * The block with FP8 GEMM operands.  The KuCoin news flash "CODA: new research
 * optimizes transformer training with GEMM epilogue programming" names FP8 in
 * section "The lazy cost of training large models" only as the reason the
 * non-GEMM share of training time grows (faster matrix products, unchanged
 * data movement); it gives no FP8 recipe.  This library's: OCP E4M3 codes
 * (max 448, no infinities), round to nearest even with saturation, one fp32
 * scale per tensor (t ~ s * decode(code)), both GEMM operands K-major, fp32
 * accumulation, and the epilogue programs of the bf16 block.  Scales live in
 * device memory so that no call synchronises with the host. */

/* Quantises a bf16 tensor src [rows, cols] to e4m3 with its own per-tensor
 * scale: amax_out = max |src|, scale_out = amax / 448 (1 if amax is 0), codes
 * = e4m3(src * (1 / scale)).  transpose = 0: dst [rows, cols]; transpose = 1:
 * dst [cols, rows] (a weight [K, N] stored K-major for the FP8 GEMMs).
 * cols % 8 == 0; with transpose, rows % 4 == 0.  amax_out and scale_out are
 * single device floats. */
coda_status_t coda_fp8_quantize(const uint16_t* src, int64_t rows, int64_t cols, int transpose, uint8_t* dst,
                                float* amax_out, float* scale_out, void* stream);

/* scale_out = amax / 448 (1 if amax is 0): the next call's scale from this
 * call's amax (delayed scaling of the block's hg8). */
coda_status_t coda_fp8_scale_from_amax(const float* amax, float* scale_out, void* stream);

/* First GEMM of the FP8 block: acc = x8 Wt8^T (e4m3 x e4m3 -> fp32), then in
 * the epilogue h = acc * sx * sw + res, partial[t, i] = sum over 128-column
 * slot t of h^2 (from the fp32 h), h_out = bf16(h),
 * hg8_out = e4m3(gamma * h / s_hg), and amax_out = max |gamma * h| over the
 * whole output (zeroed by this call, then raised by atomic max).
 * x8 [M, K], Wt8 [N, K] (the weight transposed), hg8_out [M, N] e4m3;
 * res [M, N] bf16 or NULL; gamma [N] bf16; h_out [M, N] bf16 or NULL;
 * sx, sw, s_hg, amax_out single device floats; partial [T, M] fp32.
 * N and K multiples of 16. */
coda_status_t coda_gemm_res_partialrms_fp8(const uint8_t* x8, const float* sx, const uint8_t* Wt8, const float* sw,
                                           const uint16_t* res, const uint16_t* gamma, const float* s_hg,
                                           uint16_t* h_out, uint8_t* hg8_out, float* amax_out, float* partial,
                                           int64_t M, int64_t N, int64_t K, void* stream);

/* Second GEMM of the FP8 block, with the light reduction folded in as in
 * coda_gemm_rowscale_partial: r_i = 1/sqrt(sum_t partial[t, i] / N_norm + eps),
 * out = bf16(r_i * sa * sw * (A8 Wt8^T)_ij).  A8 [M, K] e4m3 (hg8 of the first
 * GEMM), Wt8 [N, K] e4m3 (W2 transposed), sa, sw single device floats;
 * r_out [M] or NULL; out [M, N] bf16.  K a multiple of 16. */
coda_status_t coda_gemm_rowscale_partial_fp8(const uint8_t* A8, const float* sa, const uint8_t* Wt8, const float* sw,
                                             const float* partial, int64_t T, int64_t N_norm, float eps,
                                             float* r_out, uint16_t* out, int64_t M, int64_t N, int64_t K,
                                             void* stream);

/* The unfused FP8 chain the fused FP8 block is measured against:
 * coda_gemm_fp8 gives t = bf16(sa * sw * (A8 Wt8^T)) (A8 [M, K], Wt8 [N, K]
 * e4m3; K a multiple of 16); after coda_unfused_add (h = t + res),
 * coda_unfused_rmsnorm_fp8 writes y8 = e4m3(gamma * h * r / s_y) [M, N]
 * (r = 1/sqrt(mean(h^2) + eps), r_out [M] or NULL), amax_out = max |y|
 * (zeroed by the call), N a multiple of 16; then coda_gemm_fp8(y8, s_y, W2t8,
 * ...) gives out. */
coda_status_t coda_gemm_fp8(const uint8_t* A8, const float* sa, const uint8_t* Wt8, const float* sw, uint16_t* out,
                            int64_t M, int64_t N, int64_t K, void* stream);
coda_status_t coda_unfused_rmsnorm_fp8(const uint16_t* h, const uint16_t* gamma, float eps, const float* s_y,
                                       uint8_t* y8_out, float* amax_out, float* r_out, int64_t M, int64_t N,
                                       void* stream);

/* ---------------------------------------------- block-scaled e4m3 (MXFP8)
 *
 * The block with microscaled FP8 operands (the OCP "Microscaling Formats (MX)"
 * layout; the article gives no low-precision recipe, see the FP8 section):
 * every 32 consecutive elements along the reduction dimension K share one
 * power-of-two scale 2^e, stored as the byte e + 127 (E8M0); the elements are
 * e4m3 codes of v * 2^-e.  e is the smallest exponent that keeps the block's
 * largest magnitude within 448 (no element saturates), clamped to
 * [-127, 127]; an all-zero block takes e = 0.  The scales replace the FP8
 * block's per-tensor scale of hg, which had to come from an earlier call.
 *
 * Scale layouts (nkb = K / 128 k-blocks for an operand of R rows and K
 * columns, K a multiple of 128; E(i, j) = the byte of row i, 32-element
 * block j, whose k-block is kb = j / 4 and step s = j % 4).  Which layout an
 * operand takes depends on its side of the GEMM:
 *   operand 0, the left operand A: one 512-byte atom per (k-block, 128-row
 *     block), atoms kb-major (nrb = ceil(R / 128) row blocks); E(i, j) at
 *     (kb * nrb + i / 128) * 512 + (i % 32) * 16 + ((i / 32) % 4) * 4 + s.
 *   operand 1, the right operand B (stored [N, K]): one 4 KB image per
 *     (k-block, 256-row tile), images kb-major (ntl = ceil(R / 256) tiles),
 *     each tile's two atoms four times over, so that the GEMM copies the
 *     image into tensor memory at once; E(i, j) at (kb * ntl + i / 256) *
 *     4096 + ((i / 128) % 2) * 2048 + rep * 512 + (i % 32) * 16 +
 *     ((i / 32) % 4) * 4 + s for each rep = 0..3.
 * Padding rows (up to whole row blocks / tiles) hold 127.
 * coda_mx_sf_bytes(R, K, operand) = nkb * nrb * 512 (A) or nkb * ntl * 4096
 * (B); -1 for a bad shape or operand. */
int64_t coda_mx_sf_bytes(int64_t rows, int64_t cols, int operand);

/* MXFP8 codes of a row-major bf16 matrix src [rows, cols], blocked along
 * each row: q_out [rows, cols] e4m3, sf_out the scales in the layout of
 * `operand` (0: A, 1: B; coda_mx_sf_bytes(rows, cols, operand) bytes, every
 * byte written).  cols % 128 == 0.  Used for the weight W2
 * stored transposed ([N2, N], operand 1) and for the unfused chain's y
 * (operand 0). */
coda_status_t coda_mx_quantize(const uint16_t* src, int64_t rows, int64_t cols, int operand, uint8_t* q_out,
                               uint8_t* sf_out, void* stream);

/* First GEMM of the MXFP8 block: as coda_gemm_res_partialrms_fp8 (e4m3 x8
 * [M, K] and Wt8 [N, K] with per-tensor scales sx, sw; h = acc * sx * sw +
 * res; partial[t, i] over 128-column slots; h_out bf16 or NULL), except that
 * hg = gamma * h is written in MXFP8 from the epilogue: hq_out [M, N] e4m3
 * codes and hsf_out its scales in the A layout (coda_mx_sf_bytes(M, N, 0)
 * bytes; each 32-column block of a row quantised from the fp32 values as
 * they are formed).  N a multiple of 128, K of 16. */
coda_status_t coda_gemm_res_partialrms_mx(const uint8_t* x8, const float* sx, const uint8_t* Wt8, const float* sw,
                                          const uint16_t* res, const uint16_t* gamma, uint16_t* h_out,
                                          uint8_t* hq_out, uint8_t* hsf_out, float* partial, int64_t M, int64_t N,
                                          int64_t K, void* stream);

/* Second GEMM of the MXFP8 block: acc = A Wt^T with block-scaled operands
 * (tcgen05 kind::mxf8f6f4: the scales are applied inside the MMA), then as
 * coda_gemm_rowscale_partial: r_i = 1/sqrt(sum_t partial[t, i] / N_norm +
 * eps), out = bf16(r_i * acc_ij), r_out [M] or NULL.  partial == NULL gives
 * a plain MXFP8 GEMM (r = 1; T, N_norm, eps, r_out ignored).  Aq [M, K] with
 * scales Asf in the A layout, Wq [N, K] (W2 transposed) with scales Wsf in
 * the B layout; out [M, N] bf16.  N and K multiples of 128.  Launched with
 * programmatic stream serialisation after coda_gemm_res_partialrms_mx, as
 * the FP8 pair. */
coda_status_t coda_gemm_rowscale_partial_mx(const uint8_t* Aq, const uint8_t* Asf, const uint8_t* Wq,
                                            const uint8_t* Wsf, const float* partial, int64_t T, int64_t N_norm,
                                            float eps, float* r_out, uint16_t* out, int64_t M, int64_t N, int64_t K,
                                            void* stream);

/* ---------------------------------------------------------------- testing */

/* Launches one block that waits on a barrier nothing ever signals, with time
 * limit limit_ns.  The wait must give up: *gave_up_dev (device int) becomes 1
 * and the device status word records a timeout (read it with
 * coda_poll_status).  Used to test the bounded-wait path without a fault. */
coda_status_t coda_selftest_bounded_wait(int64_t limit_ns, int* gave_up_dev, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CODA_H_ */
