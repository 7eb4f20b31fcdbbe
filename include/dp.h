/*
 * dp.h -- C ABI of the displaced-patch-parallelism block step for B200 (sm_100a).
 *
 * The method is DistriFusion's displaced patch parallelism ("DistriFusion:
 * Distributed Parallel Inference for High-Resolution Diffusion Models",
 * study.space summary, Method; atlas.scime.ai summary, Approach): an image
 * latent is split into P row patches ("bands"); every band computes its own
 * rows with fresh activations and takes the context it needs from the other
 * bands out of the previous denoising step's activations.  Here all P bands
 * live on one GPU and are computed in one launch per layer; DistriFusion's
 * per-layer AllGather becomes a device-local refresh of the stale buffers.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every call returns an int status: DP_OK or one of the DP_ERR_* codes.
 *    dp_last_error() returns a message for the calling thread's last error.
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL is the legacy default stream) and never synchronises.  Kernel-side
 *    failures (a bounded wait that ran out) are recorded in a device status
 *    word that dp_device_status() reads.
 *  - The caller owns every buffer.  No call allocates, frees or keeps a
 *    pointer past its return, except that dp_block_state remembers its
 *    workspace pointer.
 *  - Device pointers must be 16-byte aligned.  Images are NHWC (row-major
 *    [H][W][C], batch 1); token matrices are row-major [T][C] with tokens in
 *    raster order of the image, so band p of an HxW image is the contiguous
 *    token range [p*T/P, (p+1)*T/P).
 *  - Bands are equal: H % P == 0 (DP_ERR_UNSUPPORTED otherwise).
 *  - Modes: DP_MODE_SYNC (warm-up step: every band sees fresh context),
 *    DP_MODE_DISPLACED (other bands' context is the stale previous step),
 *    DP_MODE_NAIVE (other bands are invisible: zero halo, own keys only).
 *  - dtype: DP_BF16 (bf16 storage, bf16 tensor-core products, fp32
 *    accumulation) or DP_FP32 (fp32 storage and fp32 arithmetic throughout;
 *    the 3x3 conv then runs on the CUDA cores).
 *    Statistics, GroupNorm scale/shift and biases are always fp32.
 */
#ifndef DP_H
#define DP_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DP_API __attribute__((visibility("default")))
#else
#define DP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define DP_OK 0
#define DP_ERR_INVALID_ARG (-1) /* null pointer, bad size, bad enum            */
#define DP_ERR_UNSUPPORTED (-2) /* shape / alignment / dtype the kernels lack   */
#define DP_ERR_STATE (-3)       /* displaced step before any step filled state  */
#define DP_ERR_CUDA (-4)        /* a CUDA runtime or driver call failed         */
#define DP_ERR_TIMEOUT (-5)     /* a device-side bounded wait ran out           */

/* step modes */
#define DP_MODE_SYNC 0
#define DP_MODE_DISPLACED 1
#define DP_MODE_NAIVE 2

/* storage types */
#define DP_BF16 0
#define DP_FP32 1

/* block kinds for dp_block_desc_init */
#define DP_BLOCK_GN_CONV 0  /* GroupNorm (+SiLU) -> 3x3 conv                                */
#define DP_BLOCK_RESBLOCK 1 /* GN -> SiLU -> conv1 -> GN -> SiLU -> conv2 -> + x / shortcut */
#define DP_BLOCK_ATTN 2     /* GN -> q,k,v proj -> stale-K/V attention -> out proj -> + x   */
#define DP_BLOCK_UNET_MINI 3 /* conv_in -> ResBlock(320) -> down -> ResBlock(320->640) ->   */
                             /* Attn(640) -> down -> ResBlock(640->1280) -> Attn(1280)      */
#define DP_BLOCK_TRANSFORMER 4 /* SDXL-shaped: GN -> proj_in -> [LN -> self-attention] + ->   */
                               /* [LN -> cross-attention] + -> [LN -> GEGLU FF] + ->          */
                               /* proj_out -> + x (dp_block_desc_set_context first)           */
#define DP_BLOCK_UNET_SDXL 5   /* SDXL-shaped U-Net step: conv_in, 3 down levels, middle,      */
                               /* 3 up levels with skips, GN -> SiLU -> conv_out               */
                               /* (dp_block_desc_set_context, _set_time_embedding first)       */

/* Message for the calling thread's last failed call ("" if none). */
DP_API const char* dp_last_error(void);

/* Library version string. */
DP_API const char* dp_version(void);

/*
 * Mode of denoising step `step` with `warmup` synchronous warm-up steps.
 * Warm-up steps run synchronously (atlas.scime.ai summary, warm-up ablation
 * rows: removing them hurts quality).  With zero warm-up, step 0 has no
 * previous step to borrow context from and runs as independent patches
 * (DP_MODE_NAIVE).  Later steps are DP_MODE_DISPLACED.
 */
DP_API int dp_mode_for_step(int step, int warmup);

/*
 * Reads and clears the library's device status word of the current device,
 * which the kernel calls below (dp_groupnorm_async ... dp_refresh_stats) set
 * when a bounded wait runs out.  The word is one per device for the whole
 * library: every such call on that device, on any stream, shares it, so a
 * DP_ERR_TIMEOUT here says that some call timed out since the last read, not
 * which.  Block steps keep a word of their own in their state (see
 * dp_block_status).  Synchronises `stream` first.  *status receives DP_OK or
 * DP_ERR_TIMEOUT.  Returns DP_ERR_CUDA if the read fails.
 */
DP_API int dp_device_status(void* stream, int* status);

/*
 * Failure-path self-test (the pages have no counterpart; it exists to test
 * the library's own failure detection).  Every pipeline wait in the library's
 * kernels is bounded by a wall-clock limit; when the limit runs out the
 * kernel records DP_ERR_TIMEOUT, drains what it has in flight and returns,
 * so the CUDA context stays usable.  This call launches one small kernel that
 * runs the same bounded-wait code on a wait nothing ever ends -- an mbarrier
 * no thread arrives at (DP_SELFTEST_WAIT_MBARRIER) or a global-memory flag no
 * thread writes (DP_SELFTEST_WAIT_FLAG) -- with a limit of `limit_us`
 * microseconds (1 .. 1000000) instead of the kernels' 2 s.  The wait runs
 * out, DP_ERR_TIMEOUT lands in the library's status word (dp_device_status
 * reads it) and the kernel returns; no copy or MMA is in flight.
 * DP_ERR_INVALID_ARG for an unknown kind or a limit out of range.
 */
#define DP_SELFTEST_WAIT_MBARRIER 0
#define DP_SELFTEST_WAIT_FLAG 1
DP_API int dp_selftest_bounded_wait(int kind, unsigned limit_us, void* stream);

/* ------------------------------------------------------------------------
 * Corrected asynchronous GroupNorm, fused with SiLU and the storage cast.
 * (atlas.scime.ai summary, Approach: "a corrected asynchronous GroupNorm";
 *  GroupNorm ablation rows: on-device-only, stale-only and synchronous
 *  statistics are the alternatives it improves on.)
 *
 * For band p and group g (C/G consecutive channels) the fresh raw moments
 * f[p][g] = (E[x], E[x^2]) over the band's rows are reduced from x.  The
 * moments each band normalises with are
 *   SYNC:       the whole-image moments, mean over bands of f;
 *   DISPLACED:  stale_global[g] + w * (f[p][g] - stale_local[p][g]);
 *   NAIVE:      f[p][g].
 * var = E[x^2] - E[x]^2; a negative corrected var falls back to the band's
 * fresh var.  Then y = (x - mean) * rsqrt(var + eps) * gamma_c + beta_c, and
 * if silu != 0, y = y * sigmoid(y); y is stored in `dtype`.
 *
 *  x            [H][W][C] dtype, device, read
 *  y            [H][W][C] dtype, device, written (may not alias x)
 *  gamma, beta  [C] fp32, device
 *  stale_global [G][2] fp32 (mean, E[x^2]), device; read in DISPLACED only
 *  stale_local  [P][G][2] fp32, device; read in DISPLACED only
 *  fresh_local  [P][G][2] fp32, device, written: f (the next step's stale_local)
 *  used_stats   [P][G][2] fp32 (mean, var), device, written
 *  workspace    device scratch of dp_groupnorm_workspace_size() bytes.  Its
 *               first 256 + 128 * P * G bytes must be zero-filled before its
 *               first use and are left zero-filled by every call that
 *               completes; the rest holds per-block partial sums and needs no
 *               initialisation.  A workspace of at least 256 + 128 * P * G
 *               bytes but smaller than the full size is accepted and runs the
 *               two-kernel path.  Calls that overlap on the GPU must not share
 *               a workspace.
 *  workspace_bytes  its size; smaller than 256 + 128 * P * G is an error.
 * Errors: DP_ERR_INVALID_ARG (null pointer, bad mode/dtype, eps <= 0, small
 * workspace), DP_ERR_UNSUPPORTED (shape limits below, unaligned x/y).
 * SiLU is h + h tanh(h), h = z/2, with the hardware tanh approximation
 * (relative error below 1e-4 before the cast, measured on B200).
 * Needs C % G == 0, C % 8 == 0 (bf16) or C % 4 == 0 (fp32), C/8 <= 1024.
 * ---------------------------------------------------------------------- */
DP_API size_t dp_groupnorm_workspace_size(int H, int W, int C, int G, int P);
DP_API int dp_groupnorm_async(const void* x, void* y, const float* gamma, const float* beta,
                       int H, int W, int C, int G, int P, float eps, float w, int silu,
                       int mode, int dtype, const float* stale_global,
                       const float* stale_local, float* fresh_local, float* used_stats,
                       void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * dp_groupnorm_async for callers that cannot allocate device memory.
 * DistriFusion has no counterpart of this call; it exists for integration only.
 *
 * Some callers have no way to obtain a workspace: code that runs where
 * cudaMalloc is off limits (it can synchronise the device, which a latency-
 * critical or real-time loop cannot afford), hosts with a fixed device-memory
 * budget granted up front, and plain C callers without a caching allocator.
 * This entry point takes the same arguments as dp_groupnorm_async minus the
 * workspace and uses a fixed scratch array inside the library instead.
 *
 *  - Limit: the scratch holds 64 KiB, enough for P * G up to 510 (bands x
 *    groups); larger requests return DP_ERR_UNSUPPORTED with a message.
 *  - Every GPU that loads the library holds those 64 KiB until the process
 *    exits.
 *  - The first call on a device looks the array's device address up
 *    (cudaGetSymbolAddress) and keeps it for the life of the process; make
 *    that first call before any stream capture.  The kept address does not
 *    survive cudaDeviceReset (or any re-creation of the device's primary
 *    context): do not call this entry point on a device after resetting it.
 *  - Each call clears the part of the scratch it uses (a cudaMemsetAsync of
 *    256 + 128 * P * G bytes on `stream`) before its kernels; nothing is
 *    allocated.
 *  - All calls share the one array and it keeps the last call's contents:
 *    calls whose kernels overlap on the GPU (different streams, no ordering)
 *    race on it and give wrong results.  Order them on one stream.
 * ---------------------------------------------------------------------- */
DP_API int dp_groupnorm_async_noalloc(const void* x, void* y, const float* gamma,
                                      const float* beta, int H, int W, int C, int G, int P,
                                      float eps, float w, int silu, int mode, int dtype,
                                      const float* stale_global, const float* stale_local,
                                      float* fresh_local, float* used_stats, void* stream);

/* ------------------------------------------------------------------------
 * 3x3 convolution, padding 1, stride 1 or 2, whose halo rows come from the
 * stale buffer (study.space summary, Method: patches reuse the previous
 * step's activations to keep their interaction).
 *
 * Output row r of band p (band = Ho/P output rows) reads input row
 * rho = stride*r + kh - 1: rho outside [0,H) is zero padding; rho inside
 * band p (band = H/P input rows) comes from a_fresh; rho in another band
 * comes from a_fresh (SYNC), a_stale (DISPLACED) or is zero (NAIVE).
 * Columns use ordinary zero padding.  out = conv + bias (+ residual).
 *
 *  a_fresh, a_stale  [H][W][Cin] dtype, device (a_stale read in DISPLACED only)
 *  weight            [Cout][3][3][Cin] dtype, device
 *  bias              [Cout] fp32, device, or NULL
 *  residual          [Ho][Wo][Cout] dtype, device, or NULL
 *  out               [Ho][Wo][Cout] dtype, device, written
 *  workspace         NULL, or device scratch of dp_gemm_workspace_size() bytes,
 *                    16-byte aligned, zero-filled before its first use (every
 *                    call leaves its counters zero).  With it, a conv with too
 *                    few output tiles to fill the GPU cuts K into runs on
 *                    separate SM pairs; each run stores an fp32 partial and
 *                    the last run of a tile sums them in run order.  Calls
 *                    that overlap on the GPU must not share it.
 * Ho = (H-1)/stride + 1.  Needs Cin % 64 == 0 (bf16) or % 16 == 0 (fp32),
 * Cout % 32 == 0 or Cout <= 16, H % P == 0, Ho % P == 0, W even when stride
 * 2.  Any W works; ragged tiles are masked.  bf16 runs on the tensor cores
 * (tcgen05, operands staged by TMA); fp32 runs in fp32 on the CUDA cores (bias
 * 16-byte aligned); Cout <= 16 (a U-Net's conv_out back to the latent's
 * channels) runs as fp32 multiply-adds on the CUDA cores for either dtype,
 * rounded once to the output type.
 * Errors: DP_ERR_INVALID_ARG (null pointers, bad mode/dtype, aliasing,
 * missing stale buffer in DISPLACED), DP_ERR_UNSUPPORTED (shape, alignment).
 * ---------------------------------------------------------------------- */
DP_API size_t dp_gemm_workspace_size(void);
DP_API int dp_conv3x3_halo(const void* a_fresh, const void* a_stale, const void* weight,
                    const float* bias, const void* residual, void* out, int H, int W,
                    int Cin, int Cout, int stride, int P, int mode, int dtype,
                    void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * The GroupNorm -> 3x3 conv pair of a block as two calls that never store the
 * normalised activations whole: dp_groupnorm_stats computes the moments each
 * band normalises with (the statistics half of dp_groupnorm_async), and
 * dp_conv3x3_halo_gn convolves GroupNorm(x) (+SiLU), normalising each input
 * tile in shared memory on its way to the tensor cores ("DistriFusion",
 * atlas.scime.ai summary, Approach: the corrected GroupNorm feeds the conv;
 * study.space summary, Method: other bands' rows are the previous step's
 * activations).
 *
 * dp_groupnorm_stats: arguments, statistics, workspace rules and errors as
 *   dp_groupnorm_async, without y, gamma, beta, eps and silu; writes
 *   fresh_local and used_stats only.
 *
 * dp_conv3x3_halo_gn: out = conv3x3(a) + bias (+ residual), stride 1, where a
 *   is x normalised per band with used_stats (scale = rsqrt(var + eps) *
 *   gamma_c, shift = beta_c - mean * scale, then SiLU if silu != 0, then the
 *   bf16 cast -- the same arithmetic as dp_groupnorm_async's output), and the
 *   halo rule of dp_conv3x3_halo: an input row of another band is a row of x
 *   normalised with that band's moments (SYNC), the row of a_stale
 *   (DISPLACED; a_stale holds normalised activations) or zero (NAIVE).
 *    x         [H][W][Cin] bf16, device: the GroupNorm's input
 *    a_stale   [H][W][Cin] bf16, device: the previous step's normalised
 *              activations; read in DISPLACED mode only, and only rows just
 *              outside a band (the first and last row of every band)
 *    a_next    [H][W][Cin] bf16, device, or NULL: receives the normalised
 *              first and last row of every band (the rows the next step's
 *              displaced call reads as its a_stale); other rows untouched.
 *              May not overlap x, a_stale, residual or out.
 *    used_stats [P][G][2] fp32 (mean, var), device (dp_groupnorm_stats)
 *    gamma, beta [Cin] fp32, device, 16-byte aligned;  weight, bias, residual, out as
 *              dp_conv3x3_halo (Ho = H, Wo = W).
 *   Needs bf16, W >= 128, Cin % 64 == 0, Cin % G == 0, Cout % 160 == 0,
 *   H % P == 0.  Tiles are one output row x 128 columns; the three input rows
 *   a tile reads are staged once per 64 input channels and the nine taps read
 *   shifted views of them.  Errors as dp_conv3x3_halo, plus DP_ERR_INVALID_ARG
 *   for null used_stats/gamma/beta, eps <= 0 or an overlapping a_next.
 * ---------------------------------------------------------------------- */
DP_API int dp_groupnorm_stats(const void* x, int H, int W, int C, int G, int P, float w, int mode,
                              int dtype, const float* stale_global, const float* stale_local,
                              float* fresh_local, float* used_stats, void* workspace,
                              size_t workspace_bytes, void* stream);
DP_API int dp_conv3x3_halo_gn(const void* x, const void* a_stale, void* a_next,
                              const float* used_stats, const float* gamma, const float* beta, int G,
                              float eps, int silu, const void* weight, const float* bias,
                              const void* residual, void* out, int H, int W, int Cin, int Cout,
                              int P, int mode, void* stream);

/* ------------------------------------------------------------------------
 * Direct 3x3 conv for few input channels (the latent input conv), same
 * halo rule and layouts as dp_conv3x3_halo, stride 1, bf16 only.
 * Needs Cin <= 16, Cout % 32 == 0.  Runs on the CUDA cores.
 * ---------------------------------------------------------------------- */
DP_API int dp_conv3x3_halo_small(const void* a_fresh, const void* a_stale, const void* weight,
                          const float* bias, void* out, int H, int W, int Cin, int Cout,
                          int P, int mode, void* stream);

/* ------------------------------------------------------------------------
 * Token projection y = x W^T + bias (+ residual), bf16, on the tensor cores:
 * the q/k/v and output projections around the attention, and the 1x1
 * shortcut conv of a ResBlock whose channels change.
 *
 *  x         [M][K] bf16, device
 *  weight    [N][K] bf16, device (an nn.Linear-style (out, in) matrix)
 *  bias      [N] fp32 or NULL;  residual [M][N] bf16 or NULL
 *  out0..2   output column ranges [0,split), [split,2*split), [2*split,3*split)
 *            go to out0, out1, out2 ([M][split] each); with split == N only
 *            out0 is used.  The fused q/k/v projection writes k and v
 *            straight into the fresh half of the caller's K/V buffers.
 *  workspace  NULL, or the split-K scratch of dp_gemm_workspace_size() bytes
 *             (same rules as for dp_conv3x3_halo).
 * Needs K % 64 == 0, split % 32 == 0, N % split == 0, N / split <= 3.
 * ---------------------------------------------------------------------- */
DP_API int dp_linear(const void* x, const void* weight, const float* bias, const void* residual,
              void* out0, void* out1, void* out2, int M, int N, int K, int split,
              void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Self-attention over stitched fresh / stale keys and values (gist.science
 * PipeFusion explainer, Problem Statement: DistriFusion keeps full-spatial K
 * and V of every layer on every device).  For a query in band p and each
 * head: softmax(q K^T * scale) V over the keys band p sees: band p's own keys
 * and values are fresh; the other bands' are fresh (SYNC), stale (DISPLACED)
 * or left out (NAIVE).
 *
 *  q, k_fresh, v_fresh, k_stale, v_stale, o   [T][heads*head_dim] bf16, device
 *  (k_stale, v_stale read in DISPLACED only; o may not alias an input)
 *  workspace   NULL, or device scratch of dp_attn_workspace_size() bytes,
 *              16-byte aligned, zero-filled before its first use (calls keep
 *              it valid).  With it the (query tile, key tile) work is split
 *              evenly over all resident CTAs, and a query tile cut between
 *              two CTAs is finished by merging their partial softmax sums
 *              through the workspace; without it each CTA takes whole query
 *              tiles.  Calls that overlap on the GPU must not share it.
 * Needs head_dim == 64, T % P == 0 and (T/P) % 128 == 0.
 * Runs on the tensor cores (tcgen05, S and O in tensor memory).
 * Errors: DP_ERR_INVALID_ARG (null q/k/v/o, bad mode, o aliasing an input,
 * missing stale K/V in DISPLACED), DP_ERR_UNSUPPORTED (shape, alignment).
 * ---------------------------------------------------------------------- */
DP_API size_t dp_attn_workspace_size(void);
DP_API int dp_attn_stale_kv(const void* q, const void* k_fresh, const void* v_fresh,
                     const void* k_stale, const void* v_stale, void* o, int T, int heads,
                     int head_dim, int P, float scale, int mode, void* workspace,
                     size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Cross-attention: Tq queries attend over Tk keys and values that every band
 * sees whole and fresh, as the text context of an SDXL transformer block
 * (the keys and values come from the prompt, not from the image, so they are
 * the same for every patch and need no stale copy).  The SDXL-shaped U-Net
 * step with cross-attention is a "next" extension; the pages do not discuss
 * it beyond naming SDXL as the model.
 *
 *  q  [Tq][heads*64] bf16, device;   k, v  [Tk][heads*64] bf16, device
 *  o  [Tq][heads*64] bf16, device, written;   o[t] = softmax(q k^T scale) v per head
 *  workspace: as for dp_attn_stale_kv (NULL: whole query tiles per CTA)
 * Needs head_dim == 64 and Tq % 256 == 0; any Tk >= 1 (a ragged last key
 * tile is masked).
 * ---------------------------------------------------------------------- */
DP_API int dp_attn_cross(const void* q, const void* k, const void* v, void* o, int Tq, int Tk,
                  int heads, int head_dim, float scale, void* workspace, size_t workspace_bytes,
                  void* stream);

/* ------------------------------------------------------------------------
 * Time-embedding term of an SDXL-shaped ResBlock ("next" item: the pages name
 * SDXL as the model; its ResBlocks add a projection of the step's time
 * embedding to the first conv's output, one vector per step that every band
 * shares, so it has no stale copy):
 *   bias[c] = conv_b[c] + temb_b[c] + sum_j temb_w[c][j] * silu(temb[j])
 * The result is the first conv's bias for the step.
 *  temb    [Ct] fp32, device;   temb_w [Cout][Ct] fp32 row-major, device;
 *  temb_b, conv_b [Cout] fp32, device, or NULL (taken as 0);
 *  bias    [Cout] fp32, device, written; may not overlap any input.
 *  1 <= Ct <= 8192, Cout >= 1.  fp32 arithmetic; asynchronous on `stream`.
 *  DP_ERR_INVALID_ARG on a null temb / temb_w / bias, bad sizes or overlap.
 * ---------------------------------------------------------------------- */
DP_API int dp_time_embedding_bias(const float* temb, const float* temb_w, const float* temb_b,
                                  const float* conv_b, float* bias, int Ct, int Cout, void* stream);

/* ------------------------------------------------------------------------
 * The sampler update between two denoising steps ("next" item: the pages'
 * results use a 50-step DDIM sampler; the update is deterministic DDIM, eta =
 * 0, of Song, Meng and Ermon, "Denoising Diffusion Implicit Models"):
 *   x_prev = sqrt(abar_prev) (x - sqrt(1 - abar_t) eps) / sqrt(abar_t)
 *            + sqrt(1 - abar_prev) eps
 * elementwise over n values; the host folds the schedule into two fp32
 * coefficients (computed in double) and the kernel does one fp32 FMA per
 * element.
 *  x, eps, x_prev  n values of `dtype` (DP_BF16 or DP_FP32), device, 16-byte
 *                  aligned; x_prev may BE x (in place) but may not otherwise
 *                  overlap x or eps.  Any n (a ragged tail is handled).
 *  abar_t, abar_prev  cumulative alpha products of the current and the
 *                  previous timestep, each in (0, 1].
 * DP_ERR_INVALID_ARG on null pointers, bad dtype, abar out of range or
 * overlap; DP_ERR_UNSUPPORTED on misalignment.  n == 0 launches nothing.
 * ---------------------------------------------------------------------- */
DP_API int dp_ddim_step(const void* x, const void* eps, void* x_prev, size_t n, double abar_t,
                        double abar_prev, int dtype, void* stream);

/* ------------------------------------------------------------------------
 * The multistep second-order DPM-Solver++ update ("next" item: the pages'
 * warm-up ablation uses a "10-step DPM-Solver"; Lu, Zhou, Bao, Chen, Li and
 * Zhu, "DPM-Solver++", the multistep second-order solver in data prediction),
 * elementwise over n values, from level abar_s to the less noisy abar_t:
 *   x0     = (x - sqrt(1 - abar_s) eps) / sqrt(abar_s)
 *   D      = x0 + (x0 - x0_prev) h / (2 (lambda_s - lambda_prev))   (2nd order)
 *   D      = x0                                  (1st order: abar_prev == 0)
 *   x_next = (sigma_t / sigma_s) x + alpha_t (1 - exp(-h)) D
 * with alpha = sqrt(abar), sigma = sqrt(1 - abar), lambda = log(alpha / sigma),
 * h = lambda_t - lambda_s; abar_t == 1 (the final step) gives x_next = x0.
 *  x, eps     n values of `dtype` (DP_BF16 or DP_FP32), device, 16-byte aligned
 *  x0_buf     n values: on entry the previous step's x0 (read only when
 *             abar_prev > 0), on exit this step's x0 for the next step
 *  x_next     n values, written; may BE x, may not otherwise overlap x, eps or
 *             x0_buf (x0_buf may not overlap any of the others)
 *  abar_prev  alpha-bar of the previous step's level (0 for a first-order step),
 *             0 < abar_prev < abar_s < abar_t <= 1 otherwise
 * The host folds the schedule into five fp32 coefficients (in double); the
 * kernel does three fp32 fused multiply-adds per element.  DP_ERR_INVALID_ARG
 * on null pointers, bad dtype, levels out of order or overlap;
 * DP_ERR_UNSUPPORTED on misalignment.  n == 0 launches nothing.
 * ---------------------------------------------------------------------- */
DP_API int dp_dpm_solver_step(const void* x, const void* eps, void* x0_buf, void* x_next, size_t n,
                              double abar_prev, double abar_s, double abar_t, int dtype, void* stream);

/* ------------------------------------------------------------------------
 * Per-token operators of an SDXL-shaped transformer block ("next" item: the
 * pages name SDXL as the model; they act on each token alone, so every band
 * runs them on its fresh tokens with no stale context).
 *
 * dp_layernorm: y[t] = (x[t] - mean_t) / sqrt(var_t + eps) * gamma + beta
 *   over the C channels of token t (biased variance).
 *   x, y [T][C] bf16, device (y may not alias x); gamma, beta [C] fp32,
 *   device.  C % 8 == 0, C <= 2048, 16-byte aligned pointers.
 * dp_geglu: y[t][c] = a * gelu(g), a = h[t][c], g = h[t][F + c], exact GELU
 *   x (1 + erf(x / sqrt 2)) / 2 (the gated feed-forward's middle step).
 *   h [T][2F] bf16, y [T][F] bf16, device, not overlapping; F % 8 == 0.
 * ---------------------------------------------------------------------- */
DP_API int dp_layernorm(const void* x, void* y, const float* gamma, const float* beta, int T,
                 int C, float eps, void* stream);
DP_API int dp_geglu(const void* h, void* y, int T, int F, void* stream);

/* ------------------------------------------------------------------------
 * The gated feed-forward's first projection with the gated GELU applied in
 * its epilogue: y[t][c] = a * gelu(g), [a | g] = x W^T + b, without storing
 * the 2F-wide projection.  W's rows (and b's entries) come interleaved in
 * blocks of 16: rows 32k..32k+15 are the value rows 16k..16k+15 and rows
 * 32k+16..32k+31 the matching gate rows (the layout of a TRANSFORMER block's
 * ff1_w and ff1_b).
 *   x [M][K] bf16, W [2F][K] bf16, b [2F] fp32 or NULL, y [M][F] bf16, device,
 *   16-byte aligned; y must not overlap x.  Needs K % 64 == 0, F % 16 == 0 and
 *   2F % 160 == 0 (the 2-SM tensor-core tiles); DP_ERR_UNSUPPORTED otherwise
 *   (a block then runs the projection and an interleaved GEGLU pass).
 * ---------------------------------------------------------------------- */
DP_API int dp_linear_geglu(const void* x, const void* weight, const float* bias, void* y, int M,
                           int F, int K, void* stream);

/* ------------------------------------------------------------------------
 * The up path of an SDXL-shaped U-Net (the pages' SDXL model, "DistriFusion",
 * atlas.scime.ai summary, Key results): each up ResBlock takes the running
 * tensor concatenated with a skip connection, and each up level ends in a
 * nearest-neighbour 2x upsample before its conv.  Both act on a pixel's own
 * rows, inside its band, so a displaced step runs them on fresh data with no
 * stale context.  Pure copies, HBM-bound.
 *
 * dp_concat_channels: out[pix] = [a[pix] | b[pix]] for npix pixels.
 *   a [npix][Ca], b [npix][Cb], out [npix][Ca + Cb], dtype (DP_BF16 or
 *   DP_FP32), device, 16-byte aligned; Ca and Cb multiples of 8 (bf16) or 4
 *   (fp32); out must not overlap a or b.  npix == 0 is a no-op.
 * dp_upsample_nearest2x: out[2i + di][2j + dj][c] = x[i][j][c], di, dj in {0, 1}.
 *   x [H][W][C], out [2H][2W][C], dtype, device, 16-byte aligned, not
 *   overlapping; C a multiple of 8 (bf16) or 4 (fp32).
 * Errors: DP_ERR_INVALID_ARG (null pointer, bad dtype or size, overlap),
 * DP_ERR_UNSUPPORTED (channel count or alignment).
 * ---------------------------------------------------------------------- */
DP_API int dp_concat_channels(const void* a, const void* b, void* out, size_t npix, int Ca, int Cb,
                              int dtype, void* stream);
DP_API int dp_upsample_nearest2x(const void* x, void* out, int H, int W, int C, int dtype,
                                 void* stream);

/* ------------------------------------------------------------------------
 * Stale-buffer refresh: the device-local replacement of DistriFusion's
 * per-layer AllGather (atlas.scime.ai summary, Approach: AllGather overlaps
 * computation; limitations: NCCL kernels take SMs).  Copies the rows of band
 * `band` (all bands if band == -1) from `fresh` to `stale`; a band is
 * rows/P rows of row_bytes bytes.  row_bytes % 16 == 0, rows % P == 0.
 * fresh and stale may not overlap.
 * ---------------------------------------------------------------------- */
DP_API int dp_refresh_stale(const void* fresh, void* stale, size_t row_bytes, int rows, int P,
                     int band, void* stream);

/*
 * Halo-only refresh.  A 3x3 conv reads other bands only at band edges: band p
 * takes the `above` rows just above its first row (the end of band p-1) and
 * the `below` rows just below its last row (the start of band p+1) from the
 * stale buffer.  For a layer whose stale buffer feeds only such a conv, this
 * copies just those rows, [(e+1) hb - above, (e+1) hb + below) for every
 * band edge e (hb = rows/P), from `fresh` to `stale`; the other rows of
 * `stale` are left as they are.  A stride-1 3x3 conv needs above = below = 1;
 * a stride-2 one with even band heights needs above = 1, below = 0.
 * Same buffer rules as dp_refresh_stale; above, below <= rows/P.  The pages
 * have no counterpart beyond the AllGather it replaces (atlas.scime.ai
 * summary, Approach): that gather sends whole patches.
 */
DP_API int dp_refresh_halo(const void* fresh, void* stale, size_t row_bytes, int rows, int P,
                    int above, int below, void* stream);

/* Statistics refresh: stale_local = fresh_local; stale_global[g] = mean over
 * bands of fresh_local[p][g].  All [.][2] fp32 device arrays. */
DP_API int dp_refresh_stats(const float* fresh_local, float* stale_local, float* stale_global,
                     int P, int G, void* stream);

/* ------------------------------------------------------------------------
 * Block step: one U-Net block over all P bands, with its cross-step state
 * (stale activations, stale K/V, stale GroupNorm statistics) held in a
 * caller-allocated device workspace.  The refresh at the end of a step is a
 * ping-pong flip of the fresh/stale halves: 0 bytes move.
 *
 * Setup:  dp_block_desc_init -> dp_block_workspace_size -> caller allocates
 *         -> dp_block_state_init (zero-fills, steps_done = 0).
 * ---------------------------------------------------------------------- */
typedef struct dp_block_desc {
  int kind;       /* DP_BLOCK_*                                   */
  int H, W;       /* image rows and columns                       */
  int C, Cout;    /* input / output channels (ATTN: Cout == C;    */
                  /* UNET_MINI: C = latent channels, Cout = 1280) */
  int G, P;       /* GroupNorm groups, bands                      */
  int heads;      /* ATTN: heads (head_dim 64)                    */
  int dtype;      /* DP_BF16 or DP_FP32 (FP32: GN_CONV only)      */
  int silu;       /* GN_CONV: SiLU after GroupNorm                */
  float eps;      /* GroupNorm epsilon                            */
  float w;        /* weight of the corrected-statistics drift term */
  int gn_stats;   /* DP_GN_STATS_*: statistics of displaced steps  */
  int ctx_len;    /* TRANSFORMER: text context tokens (Tk)        */
  int ctx_dim;    /* TRANSFORMER: text context width (Cctx)       */
  int ff_inner;   /* TRANSFORMER: feed-forward inner width (F)    */
  int temb_dim;   /* RESBLOCK: time-embedding width (0: none)     */
  int gn_fuse;    /* 1: GroupNorm -> conv through dp_conv3x3_halo_gn */
  int depth;      /* TRANSFORMER: basic transformer layers (default 1) */
  int unet_base;  /* UNET_SDXL: level widths base, 2 base, 4 base (320) */
  int unet_depth[3]; /* UNET_SDXL: transformer depth per level (0, 2, 10) */
  int ctx_fixed;  /* TRANSFORMER, UNET_SDXL: 1 = the context is the same every step */
} dp_block_desc;

/*
 * TRANSFORMER blocks: the text context's length and width and the
 * feed-forward's inner width (SDXL: 77, 2048, 4C).  The context is an input of
 * every step (the last weight pointer); it is the same for every band, so it
 * has no stale copy.  Needs ctx_len >= 1, ctx_dim % 64 == 0, ff_inner % 64 ==
 * 0.  UNET_SDXL blocks: the context of all their transformers, with
 * ff_inner 0 (each transformer's inner width is 4 C).  DP_ERR_INVALID_ARG on
 * a null descriptor or bad sizes.
 */
DP_API int dp_block_desc_set_context(dp_block_desc* d, int ctx_len, int ctx_dim, int ff_inner);

/*
 * TRANSFORMER blocks: the number of basic transformer layers (LN + self-
 * attention, LN + cross-attention, LN + feed-forward, each with its residual)
 * between the one GroupNorm / proj_in and the one proj_out (SDXL: 2 at the
 * 640-channel level, 10 at the 1280-channel level; default 1).  Every layer's
 * self-attention keeps its own stale keys and values.  1 <= depth <= 16;
 * DP_ERR_INVALID_ARG otherwise or for another kind.
 */
DP_API int dp_block_desc_set_depth(dp_block_desc* d, int depth);

/*
 * TRANSFORMER and UNET_SDXL blocks: on = 1 declares that the text context is
 * the same at every step of the state (a prompt's encoding is, for all the
 * denoising steps of one image).  Each layer's context keys and values are
 * then computed at the state's first step (steps_done == 0) and kept in the
 * workspace; later steps skip those projections (one launch per layer fewer;
 * the launch plan and dp_block_flops describe the later steps).  The caller
 * must not change the context's contents until dp_block_state_init starts a
 * new state; a changed context is not detected.  Default 0 (recomputed every
 * step).  DP_ERR_INVALID_ARG for another kind or on not in {0, 1}.
 */
DP_API int dp_block_desc_set_context_fixed(dp_block_desc* d, int on);

/*
 * UNET_SDXL blocks: one whole denoising step of an SDXL-shaped U-Net over all
 * bands (the pages' SDXL model, "DistriFusion", atlas.scime.ai summary, Key
 * results; SDXL's layout):
 *   conv_in (C -> base)
 *   down level l = 0, 1, 2 (width base << l): 2 x [ResBlock, then a
 *     transformer of depth unet_depth[l] when it is > 0]; levels 0 and 1 end
 *     in a 3x3 stride-2 conv
 *   middle: ResBlock, transformer (depth unet_depth[2], if > 0), ResBlock
 *   up level l = 2, 1, 0: 3 x [concatenate [h, skip] (the latest unused skip:
 *     the outputs of conv_in, of each down ResBlock/transformer pair and of
 *     the down convs), ResBlock, transformer as above]; levels 2 and 1 end in a
 *     nearest 2x upsample and a 3x3 conv
 *   GroupNorm -> SiLU -> conv_out (base -> C)
 * Every ResBlock adds the step's time embedding term; every transformer has
 * C/64 heads and a feed-forward inner width of 4 C; every 3x3 conv takes its
 * halo rows from the previous step's copy of its own input.  The descriptor's
 * C is the latent's channel count (even, <= 8) and Cout = C; bf16 only;
 * base % 64 == 0, base <= 512; 0 <= unet_depth[l] <= 16; H % 4P == 0,
 * W % 4 == 0, and each level's transformer needs its tokens per band to be a
 * multiple of 128.  dp_block_desc_set_context(d, Tk, Cctx, 0) and
 * dp_block_desc_set_time_embedding(d, Ct) are required.  The weight list is
 * the stages' lists in execution order (conv_in: w, b; ResBlock: its RESBLOCK
 * list without the temb vector; transformer: its TRANSFORMER list without the
 * context; down/up conv: w, b; output: gn_gamma, gn_beta, conv_w, conv_b),
 * then the step's context [Tk][Cctx] bf16 and time embedding [Ct] fp32.
 * DP_ERR_INVALID_ARG for another kind or a bad value.
 */
DP_API int dp_block_desc_set_unet(dp_block_desc* d, int base, int depth0, int depth1, int depth2);

/*
 * RESBLOCK blocks: the width Ct of the step's time embedding (0 switches it
 * off, the default).  With Ct > 0 the block takes three more weight pointers,
 * temb_w[Cout][Ct], temb_b[Cout] and the step's temb[Ct] (fp32; temb_b may be
 * NULL), and
 * adds temb_w silu(temb) + temb_b to every pixel of conv1's output (one extra
 * launch, dp_time_embedding_bias).  UNET_SDXL blocks: the width of the
 * step's time embedding every ResBlock takes (> 0 before a step).
 * DP_ERR_INVALID_ARG on a null descriptor, another kind, or Ct outside
 * [0, 8192].
 */
DP_API int dp_block_desc_set_time_embedding(dp_block_desc* d, int temb_dim);

typedef struct dp_block_state {
  void* workspace;        /* device memory of dp_block_workspace_size() bytes */
  size_t workspace_bytes;
  int cur;                /* which half of each ping-pong pair is stale       */
  int steps_done;         /* steps completed since dp_block_state_init        */
} dp_block_state;

DP_API int dp_block_desc_init(dp_block_desc* d, int kind, int H, int W, int C, int Cout, int G,
                       int P, int heads, int dtype, int silu, float eps, float w);

/*
 * GroupNorm statistics of the displaced steps of a block: the method's
 * corrected asynchronous statistics, or one of the alternatives its GroupNorm
 * ablation compares ("DistriFusion", atlas.scime.ai summary, Approach and the
 * GroupNorm ablation rows: statistics of the device's own patch only, stale
 * statistics only, and a synchronous exact pass).  Only DISPLACED steps are
 * affected; SYNC and NAIVE steps keep their own statistics.  The halo rows
 * and the keys and values stay stale in every variant.
 *   DP_GN_STATS_CORRECTED  stale_global + w (fresh_local - stale_local)  (default)
 *   DP_GN_STATS_LOCAL      the band's own fresh moments
 *   DP_GN_STATS_STALE      the previous step's whole-image moments (w = 0)
 *   DP_GN_STATS_SYNC       the exact whole-image moments of this step
 * dp_block_desc_init sets DP_GN_STATS_CORRECTED.  Returns DP_ERR_INVALID_ARG
 * for an unknown variant or a null descriptor.
 */
#define DP_GN_STATS_CORRECTED 0
#define DP_GN_STATS_LOCAL 1
#define DP_GN_STATS_STALE 2
#define DP_GN_STATS_SYNC 3
DP_API int dp_block_desc_set_gn_stats(dp_block_desc* d, int variant);

/*
 * GN_CONV and RESBLOCK blocks (and the mini U-Net's ResBlocks): with on = 1,
 * every GroupNorm -> 3x3 conv pair whose shapes dp_conv3x3_halo_gn takes runs
 * as dp_groupnorm_stats + dp_conv3x3_halo_gn, so the normalised activations
 * are never stored whole and the state keeps only their band-edge rows.  Off
 * (0) by default: on B200 the separate GroupNorm pass plus the plain conv is
 * the faster pair at the SDXL shapes (the fused conv redoes the normalisation
 * for each of the three row windows that read an input row, and its
 * shared-memory traffic slows the tensor core's operand reads).
 * DP_ERR_INVALID_ARG for a null descriptor or on not 0/1.
 */
DP_API int dp_block_desc_set_gn_fusion(dp_block_desc* d, int on);
DP_API size_t dp_block_workspace_size(const dp_block_desc* d);
DP_API int dp_block_state_init(const dp_block_desc* d, dp_block_state* s, void* workspace,
                        size_t workspace_bytes, void* stream);

/*
 * Runs one step of the block in `mode` and then refreshes the state.
 *  x    block input, [H][W][C] dtype, device (ATTN: the same image as tokens)
 *  out  block output, [H][W][Cout] dtype, device (may not alias x)
 *  weights: device pointers, in this order per kind --
 *   GN_CONV:  gn_gamma[C], gn_beta[C], conv_w[Cout][3][3][C], conv_b[Cout]
 *   RESBLOCK: gn1_gamma[C], gn1_beta[C], conv1_w[Cout][3][3][C], conv1_b[Cout],
 *             gn2_gamma[Cout], gn2_beta[Cout], conv2_w[Cout][3][3][Cout],
 *             conv2_b[Cout], then if C != Cout: short_w[Cout][C], short_b[Cout],
 *             then if temb_dim > 0: temb_w[Cout][temb_dim], temb_b[Cout] and the
 *             step's time embedding temb[temb_dim] (fp32; temb_b may be NULL)
 *   ATTN:     gn_gamma[C], gn_beta[C], wqkv[3C][C] (the q, k and v (out, in)
 *             matrices stacked), bqkv[3C], wo[C][C], bo[C]
 *   TRANSFORMER (C == heads * 64, (H*W/P) % 128 == 0, (H*W) % 256 == 0):
 *             gn_gamma[C], gn_beta[C], proj_in_w[C][C], proj_in_b[C], then for each
 *             of the `depth` layers: ln1_g[C], ln1_b[C], wqkv[3C][C], bqkv[3C],
 *             wo[C][C], bo[C], ln2_g[C], ln2_b[C], cq_w[C][C], ckv_w[2C][Cctx]
 *             (the context's k and v matrices stacked), co_w[C][C], co_b[C],
 *             ln3_g[C], ln3_b[C], ff1_w[2F][C] and ff1_b[2F] (value and gate
 *             rows interleaved in blocks of 16, as dp_linear_geglu takes them:
 *             the block fuses the gated GELU into ff1 when dp_linear_geglu's
 *             shape rule holds and otherwise runs ff1 and a GEGLU pass over the
 *             same layout), ff2_w[C][F], ff2_b[C]; then proj_out_w[C][C],
 *             proj_out_b[C], and the step's context [ctx_len][ctx_dim] bf16
 *             (7 + 18 depth pointers; matrices bf16, vectors fp32; the biases may
 *             be NULL)
 *   UNET_MINI (latent [H][W][C], C even <= 16, H % 4P == 0, W % 4 == 0; output
 *             [H/4][W/4][1280]): conv_in_w[320][3][3][C], conv_in_b[320], the
 *             RESBLOCK list for 320->320 at HxW, down1_w[320][3][3][320],
 *             down1_b[320], the RESBLOCK list for 320->640 at H/2 x W/2, the ATTN
 *             list for 640 (10 heads), down2_w[640][3][3][640], down2_b[640], the
 *             RESBLOCK list for 640->1280 at H/4 x W/4, the ATTN list for 1280
 *             (20 heads) -- dp_block_weight_count() pointers in all.  Every 3x3
 *             conv of the chain (conv_in and the two stride-2 downsamplers
 *             included) takes its halo rows from the previous step's copy of its
 *             own input.
 *  Weight matrices are `dtype`; gamma, beta and biases fp32 (biases may be NULL).
 * Returns DP_ERR_STATE for DISPLACED before any completed step.
 */
DP_API int dp_block_step(const dp_block_desc* d, dp_block_state* s, const void* x, void* out,
                  const void* const* weights, int n_weights, int mode, void* stream);

/*
 * Reads and clears the block state's own device status word: the kernels of
 * this state's dp_block_step calls record a bounded wait that ran out there
 * (DP_ERR_TIMEOUT), so blocks stepped on different streams can tell whose
 * step timed out.  Synchronises `stream` first; *status receives DP_OK or
 * DP_ERR_TIMEOUT.  DP_ERR_INVALID_ARG on a null or uninitialised state.
 */
/*
 * Block steps as CUDA graphs (a step of a large block is hundreds of launches;
 * replaying them as one graph removes their host-side launch cost and part of
 * the gaps between them).  dp_block_graph_create captures one step of `d` in
 * `mode` for each ping-pong parity, on the caller's (non-default) `stream`,
 * with the given x, out and weight pointers fixed in the graphs; nothing runs
 * and the state does not change.  dp_block_graph_launch then runs the step of
 * the state's current parity on `stream`, flips the parity and counts the
 * step, exactly as dp_block_step with those arguments would: new inputs are
 * copied into the captured x before a launch, and anything the caller does
 * between steps (a sampler update) runs between launches.
 *   - Capture after the state's first step (DP_ERR_STATE before it): the
 *     graphs are later steps (a fixed context's keys and values, computed at
 *     the first step, are not in them).
 *   - A graph runs only on the state it was captured on (DP_ERR_INVALID_ARG
 *     otherwise) and while the weights, x, out and workspace stay where they
 *     were at capture.
 *   - DP_ERR_CUDA if the capture or instantiation fails; nothing is left
 *     allocated then.  dp_block_graph_destroy frees the graphs (NULL is a no-op).
 * Handles are opaque and owned by the caller; one handle per state at a time
 * and stream order between its launches and other calls on the state.
 */
typedef struct dp_block_graph dp_block_graph;
DP_API int dp_block_graph_create(const dp_block_desc* d, dp_block_state* s, const void* x, void* out,
                                 const void* const* weights, int n_weights, int mode, void* stream,
                                 dp_block_graph** graph);
DP_API int dp_block_graph_launch(dp_block_graph* graph, dp_block_state* s, void* stream);
DP_API int dp_block_graph_destroy(dp_block_graph* graph);

DP_API int dp_block_status(const dp_block_desc* d, const dp_block_state* s, void* stream,
                           int* status);

/* Kernel kinds reported by dp_block_launch_info. */
#define DP_KERNEL_GN_STATS 0   /* GroupNorm statistics pass                     */
#define DP_KERNEL_GN_APPLY 1   /* GroupNorm apply pass                          */
#define DP_KERNEL_GN_FUSED 2   /* single-pass GroupNorm (tensor fits on chip)   */
#define DP_KERNEL_CONV 3       /* 3x3 halo conv (tensor cores)                  */
#define DP_KERNEL_LINEAR 4     /* projection / 1x1 conv (tensor cores)          */
#define DP_KERNEL_ATTN 5       /* stale-K/V attention (tensor cores)            */
#define DP_KERNEL_COPY 6       /* device copy                                   */
#define DP_KERNEL_CONV_SMALL 7 /* direct 3x3 conv for few input channels        */
#define DP_KERNEL_SPLITK_FINISH 8 /* sum of split-K partials + bias + residual   */
#define DP_KERNEL_GN_CLUSTER 9  /* GroupNorm, one thread-block cluster per band */
#define DP_KERNEL_LAYERNORM 10  /* per-token LayerNorm                          */
#define DP_KERNEL_GEGLU 11      /* gated GELU unit of the feed-forward          */
#define DP_KERNEL_TEMB 12       /* time-embedding bias of a ResBlock's conv1     */
#define DP_KERNEL_CONV_GN 13    /* 3x3 conv of GroupNorm(x), normalised in-kernel */
#define DP_KERNEL_CONV_F32 14   /* 3x3 halo conv in fp32 on the CUDA cores       */
#define DP_KERNEL_CONV_NARROW 15 /* 3x3 halo conv to <= 16 channels, CUDA cores  */
#define DP_KERNEL_CONCAT 16     /* channel concatenation [h, skip]               */
#define DP_KERNEL_UPSAMPLE 17   /* nearest-neighbour 2x upsampling               */

/*
 * Number of kernel launches one displaced dp_block_step makes for this
 * descriptor.  A GroupNorm is one launch when its tensor fits in the GPU's
 * shared memory and two (statistics, apply) otherwise; a GroupNorm that feeds
 * a 3x3 conv dp_conv3x3_halo_gn can take (bf16, W >= 128, Cin % 64 == 0,
 * Cout % 160 == 0) is its statistics pass alone, and the conv that follows
 * normalises its own input (DP_KERNEL_CONV_GN).  Launch order --
 *   GN_CONV:  GN, conv
 *   RESBLOCK: GN1, conv1, GN2, [1x1 shortcut if C != Cout], conv2
 *             (each GN and conv a statistics pass and a CONV_GN when fused)
 *   ATTN:     GN, q/k/v projection, attention, out projection
 *   UNET_MINI: input copy, conv_in, then its blocks and downsamplers in order
 *   TRANSFORMER: GN, proj_in, then per layer LN, q/k/v projection, attention,
 *             out projection, LN, query projection, context k/v projection,
 *             cross-attention, out projection, LN, ff1, GEGLU, ff2; then proj_out
 * Negative status on a bad descriptor.
 */
DP_API int dp_block_launch_count(const dp_block_desc* d);

/*
 * Kind (DP_KERNEL_*), algorithmic flops and algorithmic bytes of launch i of
 * one dp_block_step in `mode`, from the same code path that makes the
 * launches.  Bytes count each tensor a kernel must read or write once.
 */
DP_API int dp_block_launch_info(const dp_block_desc* d, int mode, int i, int* kind,
                                double* flops, double* bytes);

/*
 * dp_block_step that also records events[i] (cudaEvent_t, passed as void*)
 * on `stream` just before its i-th kernel launch and events[n] after the
 * last, n = dp_block_launch_count(d); n_events must be >= n + 1.  The
 * elapsed time between events[i] and events[i+1] is launch i's duration.
 */
DP_API int dp_block_step_timed(const dp_block_desc* d, dp_block_state* s, const void* x, void* out,
                               const void* const* weights, int n_weights, int mode, void* stream,
                               void* const* events, int n_events);

/* Number of weight pointers dp_block_step expects for this descriptor. */
DP_API int dp_block_weight_count(const dp_block_desc* d);

/* Algorithmic FLOPs of one block step (multiply-adds count 2). */
DP_API double dp_block_flops(const dp_block_desc* d);

#ifdef __cplusplus
}
#endif

#endif /* DP_H */
