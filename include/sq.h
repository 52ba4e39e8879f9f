/*
 * sq.h -- C ABI of the B200 (sm_100a) smoothed W8A8 linear layer.
 *
 * The layer is SmoothQuant's: an activation absmax over calibration tokens,
 * the smoothing factors of eq. (4), an offline fold of those factors into the
 * weights (then per-output-channel symmetric INT8) and into the preceding
 * LayerNorm, a runtime fused LayerNorm + smoothing + symmetric INT8
 * activation quantizer, and an INT8 x INT8 -> INT32 GEMM on the tcgen05 tensor
 * cores whose epilogue dequantizes by act_scale[token] * w_scale[out].
 *
 * Sources, cited by tag below:
 *   [explainer] "SmoothQuant 如何解决激活量化难题？为什么适合 W8A8？"
 *   [review]    "SmoothQuant：大型语言模型的精准高效训练后量化 — 深度技术评审"
 *   [embedded]  "嵌入式 SLM 动态权重量化：SmoothQuant 激活异常值迁移与 INT8 部署实战"
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.   Every tensor pointer is DEVICE memory owned by the caller,
 *           contiguous, row-major, and 16-byte aligned.  The library
 *           allocates no device memory; the only library-owned device state
 *           is one status word per device (a static __device__ variable).
 * Layouts.  X is [T,K] (token, input channel).  W and Wq are [N,K]
 *           (output channel, input channel), i.e. K-major, the transpose of
 *           the review's W in Y = XW.  Y is [M,N].
 * Shapes.   K (the input width) must be a multiple of 16 in [16, 133136];
 *           the upper bound keeps 127*127*K below 2^31 so the INT32
 *           accumulators cannot overflow.  T, M or N equal to 0 is an empty
 *           problem: the call returns SQ_OK and launches nothing.  Negative
 *           sizes are SQ_ERR_SHAPE.
 * Streams.  Work is enqueued on `stream` (NULL = the legacy default stream)
 *           and every call is asynchronous.  Argument checks run on the host
 *           before anything is enqueued: on any error nothing is launched
 *           and the outputs are untouched.
 * Errors.   A launch failure returns SQ_ERR_CUDA.  Faults detected on the
 *           device (a bounded wait that ran out) are recorded in the device
 *           status word and reported by sq_sync_status().  sq_last_error()
 *           gives a one-line description of the last host-side error on the
 *           calling thread.
 * Numerics. The fp32 operations of every step run in a fixed order with one
 *           IEEE rounding each (no contraction into FMA except where stated),
 *           so integer codes, scales and INT32 accumulators are reproducible
 *           bit for bit: Delta(a) = max(a, 1e-7f) / 127; Q(v; Delta) =
 *           clamp(round_half_even(v * (1/Delta)), -127, 127), NaN -> 0.
 * Threads.  The entry points keep no host state between calls and may be
 *           called from several host threads at once.
 */
#ifndef SQ_H
#define SQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SQ_OK = 0,
  SQ_ERR_INVALID_ARG = 1, /* NULL where a tensor is required, bad enum, alpha outside [0,1] */
  SQ_ERR_SHAPE = 2,       /* K not a multiple of 16 or outside [16,133136]; negative size */
  SQ_ERR_ALIGN = 3,       /* a tensor pointer is not 16-byte aligned */
  SQ_ERR_DTYPE = 4,       /* unsupported element type for this argument */
  SQ_ERR_UNSUPPORTED = 5, /* no sm_100 device, or a size this build cannot serve */
  SQ_ERR_CUDA = 6,        /* a CUDA runtime call failed */
  SQ_ERR_TIMEOUT = 7,     /* device side: a bounded wait ran out (from sq_sync_status) */
  SQ_ERR_WORKSPACE = 8,   /* workspace NULL or smaller than sq_gemm_workspace_bytes() */
  SQ_ERR_BOUNDS = 9       /* device side, bounds-checked builds only: an index outside its
                             tensor was caught and that access skipped (from sq_sync_status) */
} sq_status;

typedef enum { SQ_F32 = 0, SQ_BF16 = 1 } sq_dtype;

/* Activation quantization granularity ([review] §2.5, §2.6 Fig. 3, §6.3):
 * per-tensor with a static step fixed at calibration (SmoothQuant-O3),
 * per-token with a step computed from each token's peak at run time (O1),
 * or per-tensor with one step computed at run time from the peak of the
 * whole call's activations (O2). */
typedef enum {
  SQ_ACT_PER_TENSOR_STATIC = 0,
  SQ_ACT_PER_TOKEN_DYNAMIC = 1,
  SQ_ACT_PER_TENSOR_DYNAMIC = 2
} sq_act_gran;

typedef struct CUstream_st* sq_stream; /* a cudaStream_t */

/*
 * sq_calib_absmax -- per-input-channel activation peak over calibration
 * tokens ([explainer] §四: record each input channel's activation peak on a
 * calibration set; [review] §5.3: max|X_j| in eq. (4)).
 *
 *   amax[k] = max(amax[k], max_t |f(X)[t,k]|)
 *
 * f is the identity when ln_gamma is NULL.  Otherwise f is the LayerNorm that
 * precedes the linear, with the ORIGINAL (unfolded) parameters:
 * f(X)[t,k] = ((X[t,k] - mu_t) * rstd_t) * gamma[k] + beta[k], mu_t and the
 * variance summed in the library's fixed order (128 slots of 8-element
 * chunks), rstd_t = 1 / sqrt(var_t + ln_eps).  ln_beta may be NULL (= 0).
 *
 *   x      [T,K] of type xt (SQ_F32 or SQ_BF16), read only.
 *   amax   [K] fp32, read and updated in place (a running maximum): zero it
 *          before the first batch; calling again with the next batch of
 *          tokens continues the same statistic.
 * Values must be finite.
 */
sq_status sq_calib_absmax(const void* x, sq_dtype xt, int64_t T, int64_t K,
                          const float* ln_gamma, const float* ln_beta,
                          float ln_eps, float* amax, sq_stream stream);

/*
 * sq_calib_absmax_rms -- sq_calib_absmax through an RMSNorm instead of a
 * LayerNorm (the norm of models whose smoothing fold is gamma / s alone:
 * the fold of [embedded] §二 without a beta; the pages define no RMSNorm, so
 * the reduction order below is this library's):
 *
 *   ms = mean_k x[t,k]^2 in the LayerNorm's slot order (each slot updated by
 *        one fused multiply-add), rstd = 1 / sqrt(ms + eps),
 *   amax[k] = max(amax[k], max_t |(x[t,k] * rstd) * gamma[k]|).
 *
 *   gamma [K] fp32 (required); eps finite, >= 0.  Arguments, layouts and
 *   errors otherwise as sq_calib_absmax.
 */
sq_status sq_calib_absmax_rms(const void* x, sq_dtype xt, int64_t T, int64_t K,
                              const float* gamma, float eps, float* amax,
                              sq_stream stream);

/*
 * sq_smooth_scales -- smoothing factors of eq. (4) ([review] §5.3;
 * [explainer] §三):
 *
 *   s_k = max|X_k|^alpha / max|W_k|^(1-alpha)
 *
 * max|W_k| = max_n |W[n,k]| is computed here from w [N,K] (type wt) and
 * floored at 1e-7; the ratio is evaluated in fp64 (alpha = 0.5 with square
 * roots, alpha in {0,1} without pow) and rounded once to fp32, then
 * s_k = max(s_k, 1e-4f) and inv_s_k = 1/s_k (fp32 division).
 *
 *   amax_x            [K] fp32 calibration peaks (from sq_calib_absmax).
 *   s, inv_s          [K] fp32 outputs.  s is also used as scratch.
 *   act_delta_static  [1] fp32 output or NULL: the static per-tensor step of
 *                     the smoothed activation, Delta(max_k amax_x[k]/s_k)
 *                     (the calibration peak of X diag(s)^-1, [review] §6.4).
 *   alpha             migration strength in [0, 1].
 */
sq_status sq_smooth_scales(const float* amax_x, const void* w, sq_dtype wt,
                           int64_t N, int64_t K, float alpha, float* s,
                           float* inv_s, float* act_delta_static,
                           sq_stream stream);

/*
 * sq_weight_colmax and sq_smooth_scales_peaks -- sq_smooth_scales in two
 * steps, for callers that keep the weight peaks (an alpha search, a model
 * whose weights do not change) or compute them concurrently with the
 * calibration (they do not depend on it):
 *
 *   sq_weight_colmax:        amax_w[k] = max_n |W[n,k]|   (w [N,K] type wt;
 *                            amax_w [K] fp32 out, overwritten)
 *   sq_smooth_scales_peaks:  s, inv_s (and act_delta_static) from amax_x and
 *                            amax_w exactly as sq_smooth_scales computes them
 *                            (amax_w is floored at 1e-7 there, not here)
 *
 * Arguments and errors as sq_smooth_scales; the two steps give the same
 * bits as the one call.
 */
sq_status sq_weight_colmax(const void* w, sq_dtype wt, int64_t N, int64_t K,
                           float* amax_w, sq_stream stream);
sq_status sq_smooth_scales_peaks(const float* amax_x, const float* amax_w,
                                 int64_t K, float alpha, float* s,
                                 float* inv_s, float* act_delta_static,
                                 sq_stream stream);

/*
 * sq_fuse_weights_q8 -- offline fold of s ([embedded] §二; [review] §5.1
 * eq. (3), §5.5):
 *
 *   W_hat[n,k] = W[n,k] * s_k                     (fp32)
 *   w_scale[n] = Delta(max_k |W_hat[n,k]|)        (per output channel)
 *   wq[n,k]    = Q(W_hat[n,k]; w_scale[n])        (int8, K-major)
 *   gamma_out  = gamma / s,  beta_out = beta / s  (LayerNorm fold)
 *
 *   w      [N,K] type wt; s [K] fp32; wq [N,K] int8 out; w_scale [N] fp32 out.
 *   gamma/gamma_out and beta/beta_out are optional pairs ([K] fp32 each):
 *   a pair is folded when both of its pointers are non-NULL.
 */
sq_status sq_fuse_weights_q8(const void* w, sq_dtype wt, int64_t N, int64_t K,
                             const float* s, int8_t* wq, float* w_scale,
                             const float* gamma, const float* beta,
                             float* gamma_out, float* beta_out,
                             sq_stream stream);

/*
 * sq_fold_into_producer -- fold 1/s into the linear that produces this
 * layer's input instead of into a norm or the quantizer ([review] §5.5: the
 * smoothing factor folds into the previous layer's parameters).  The
 * producer's output channel k is this layer's input channel k and has its
 * own per-output-channel scale (from sq_fuse_weights_q8 on the producer) and
 * bias, so
 *
 *   w_scale[k] = w_scale[k] / s[k],   bias[k] = bias[k] / s[k]
 *
 * (one fp32 division each, in place) makes the producer emit X diag(s)^-1
 * directly (a ReLU in between commutes, s > 0), and this layer's quantizer
 * then takes inv_s = NULL.  s [K] fp32 (from sq_smooth_scales of this
 * layer); w_scale [K] fp32 in/out; bias [K] fp32 in/out or NULL; all device
 * memory, 16-byte aligned.  Errors: SQ_ERR_SHAPE (K < 0),
 * SQ_ERR_INVALID_ARG / SQ_ERR_ALIGN for the pointers; K = 0 does nothing.
 */
sq_status sq_fold_into_producer(const float* s, int64_t K, float* w_scale,
                                float* bias, sq_stream stream);

/*
 * sq_ln_smooth_quant_act -- runtime fused LayerNorm + smoothing + symmetric
 * INT8 activation quantizer ([embedded] §二: the modified LayerNorm emits the
 * smoothed activation, which is quantized per tensor and fed to the INT8
 * GEMM; [review] §2.2, §2.5, §2.6, §6.3).
 *
 *   y = LN(x) with the folded gamma_s, beta_s (same order as sq_calib_absmax)
 *       when gamma_s != NULL (inv_s must then be NULL: s is already folded
 *       into gamma_s and beta_s), else y = x * inv_s (inv_s NULL: y = x);
 *   SQ_ACT_PER_TOKEN_DYNAMIC: act_scale[t] = Delta(max_k |y[t,k]|) (output,
 *       [T] fp32), xq[t,k] = Q(y[t,k]; act_scale[t]);
 *   SQ_ACT_PER_TENSOR_STATIC: act_scale[0] is the calibrated step (input),
 *       xq[t,k] = Q(y[t,k]; act_scale[0]); values above it saturate.
 *   SQ_ACT_PER_TENSOR_DYNAMIC: act_scale[0] = Delta(max_{t,k} |y[t,k]|)
 *       (output, [1] fp32; NaN elements are skipped by the peak and code to
 *       0), xq[t,k] = Q(y[t,k]; act_scale[0]).  Two passes over x: the peak
 *       is accumulated in act_scale[0] itself, which holds the peak, not a
 *       step, until the call's last kernel has run on the stream.
 *
 *   x [T,K] type xt; xq [T,K] int8 out.
 *   n_clipped: NULL, or an int64 counter in device memory to which the number
 *   of saturated codes is ADDED (the saturation rate of a static scale).
 */
sq_status sq_ln_smooth_quant_act(const void* x, sq_dtype xt, int64_t T,
                                 int64_t K, const float* gamma_s,
                                 const float* beta_s, float ln_eps,
                                 const float* inv_s, sq_act_gran gran,
                                 float* act_scale, int8_t* xq,
                                 int64_t* n_clipped, sq_stream stream);

/*
 * sq_rms_smooth_quant_act -- the runtime quantizer behind an RMSNorm whose
 * gamma carries the folded 1/s (gamma_s = gamma / s, from
 * sq_fuse_weights_q8 with beta NULL):
 *
 *   y[t,k] = (x[t,k] * rstd_t) * gamma_s[k]   (rstd as sq_calib_absmax_rms)
 *
 * then quantized at granularity gran exactly as sq_ln_smooth_quant_act
 * (per-token dynamic, per-tensor static, per-tensor dynamic).  gamma_s [K]
 * fp32 (required).  Arguments, layouts and errors otherwise as
 * sq_ln_smooth_quant_act.
 */
sq_status sq_rms_smooth_quant_act(const void* x, sq_dtype xt, int64_t T,
                                  int64_t K, const float* gamma_s, float eps,
                                  sq_act_gran gran, float* act_scale,
                                  int8_t* xq, int64_t* n_clipped,
                                  sq_stream stream);

/*
 * sq_gemm_workspace_bytes -- device scratch sq_gemm_w8a8 needs for this
 * shape on the current device (0 when it needs none).  Problems of up to 8
 * tokens, and of up to 128 tokens whose output is too narrow for 128-row
 * tiles to give every SM one (N / 192 or N / 256 below the SM count), take
 * the stream-K weight-streaming path.  It splits the K loop of a weight tile
 * across SMs and reduces the exact INT32 partial tiles in the workspace:
 * 256 bytes per 128 output channels (rounded up to 256) plus
 * 2 * M * 128 * 4 bytes per SM used.  Every other shape needs none.
 */
size_t sq_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * sq_gemm_w8a8 -- INT8 GEMM with dequantizing epilogue ([review] §2.6 Fig. 3:
 * scales only on the outer dimensions; [embedded] §三: integer inner product,
 * then one float rescale per output):
 *
 *   acc[t,n] = sum_k xq[t,k] * wq[n,k]                 (exact INT32)
 *   y[t,n]   = (float)acc[t,n] * (as_t * w_scale[n])   (fp32, RNE)
 *   as_t     = act_scale[t] if act_per_token else act_scale[0]
 *
 *   xq [M,K] int8; wq [N,K] int8; w_scale [N] fp32;
 *   y  [M,N] of type yt (SQ_F32, or SQ_BF16 = RNE of the fp32 value);
 *   acc_out: NULL, or [M,N] int32 that receives the accumulators.
 *   workspace: at least sq_gemm_workspace_bytes(M,N,K) bytes of device
 *   memory, 16-byte aligned (may be NULL when that size is 0).  It needs no
 *   initialization: each call zeroes the part it counts with and overwrites
 *   the rest.  Calls that share a workspace must not run concurrently.
 */
sq_status sq_gemm_w8a8(const int8_t* xq, const int8_t* wq, int64_t M,
                       int64_t N, int64_t K, const float* act_scale,
                       int act_per_token, const float* w_scale, void* y,
                       sq_dtype yt, int32_t* acc_out, void* workspace,
                       size_t workspace_bytes, sq_stream stream);

/*
 * sq_gemm_w8a8_bias -- sq_gemm_w8a8 followed by the linear's bias: the
 * smoothing leaves a bias untouched ([review] §5.1 eq. (3): X W + b =
 * (X diag(s)^-1)(diag(s) W) + b), so it is added to the dequantized output:
 *
 *   y[t,n] = (float)acc[t,n] * (as_t * w_scale[n]) + bias[n]
 *
 * as one more fp32 addition (never fused with the multiply), before the bf16
 * conversion.  bias: [N] fp32 device memory, 16-byte aligned, or NULL (then
 * identical to sq_gemm_w8a8).  All other arguments, errors and the workspace
 * as for sq_gemm_w8a8.
 */
sq_status sq_gemm_w8a8_bias(const int8_t* xq, const int8_t* wq, int64_t M,
                            int64_t N, int64_t K, const float* act_scale,
                            int act_per_token, const float* w_scale,
                            const float* bias, void* y, sq_dtype yt,
                            int32_t* acc_out, void* workspace,
                            size_t workspace_bytes, sq_stream stream);

/*
 * sq_gemm_w8a8_noalloc -- sq_gemm_w8a8 for callers that cannot allocate
 * device memory.  (No counterpart on the pages: this is a property of the
 * library interface, not of the method.)
 *
 * Some callers cannot call cudaMalloc or hand out a workspace: code running
 * inside an engine or framework that owns every device allocation and
 * forbids new ones while it executes, or plugin-style hooks whose execute
 * step receives only its inputs and outputs.  This entry point takes the
 * same arguments as sq_gemm_w8a8 minus the workspace and allocates nothing
 * (no cudaMalloc/cudaFree, no allocating library routine): the scratch the
 * stream-K path needs lives in a fixed array of 8 MiB (8,388,608 bytes) of
 * device memory that the library reserves on every GPU that loads it, held
 * until the process exits.
 *
 *   - A shape is refused with SQ_ERR_WORKSPACE, before anything is
 *     launched, exactly when sq_gemm_workspace_bytes(M,N,K) > 8,388,608.
 *     On the stream-K path that size is the tile counters (4 bytes per 128
 *     output channels, rounded up to 256) plus G * 2 * M * 512 bytes, G =
 *     min(SM count, 128-channel tiles x 128-byte k-blocks); with G = 148 the
 *     largest M served is 55.  Shapes off that path need no scratch and are
 *     always served.
 *   - The first call on a device looks up the array's device address with
 *     cudaGetSymbolAddress, so make that first call before any stream capture
 *     begins on that device.
 *   - Every call on a device uses the same array, and each call resets the
 *     part of it that must start at zero.  Calls whose executions overlap on
 *     the GPU (different streams, or different host threads) race on it and
 *     give wrong results: serialize them.
 */
sq_status sq_gemm_w8a8_noalloc(const int8_t* xq, const int8_t* wq, int64_t M,
                               int64_t N, int64_t K, const float* act_scale,
                               int act_per_token, const float* w_scale,
                               void* y, sq_dtype yt, int32_t* acc_out,
                               sq_stream stream);

/*
 * sq_bmm_w8a8 -- batched INT8 matrix multiplication for the attention block
 * (SmoothQuant quantizes the batched matmuls of attention to INT8 as well,
 * [review] §5.6 Fig. 6): for every b in [0, batch)
 *
 *   acc[b,t,n] = sum_k xq[b,t,k] * wq[b,n,k]                (exact INT32)
 *   y[b,t,n]   = (float)acc[b,t,n] * (as * ws)               (fp32, RNE)
 *   as = act_scale[b*M + t] if act_per_token else act_scale[b]
 *   ws = w_scale[b*N + n]   if w_per_channel else w_scale[b]
 *
 * e.g. scores = Q K^T with xq = Q [heads, T, d] and wq = K [heads, T, d],
 * or P V with xq = P [heads, T, T] and wq = V^T [heads, d, T].  Both
 * operands are K-major (K contiguous, a multiple of 16); the batches are
 * stored back to back: xq [batch, M, K], wq [batch, N, K], y and acc_out
 * [batch, M, N].  One persistent tcgen05 launch covers every batch.
 * No workspace.  Errors as sq_gemm_w8a8 (no bias); batch times the number
 * of 128 x 128 tiles must stay below 2^31.
 */
sq_status sq_bmm_w8a8(const int8_t* xq, const int8_t* wq, int64_t batch,
                      int64_t M, int64_t N, int64_t K, const float* act_scale,
                      int act_per_token, const float* w_scale,
                      int w_per_channel, void* y, sq_dtype yt, int32_t* acc_out,
                      sq_stream stream);

/*
 * sq_alpha_sweep -- choose the migration strength alpha by the layer's
 * output error (eq. (4)'s alpha, [review] §5.3; the paper sweeps it and
 * finds a sweet spot between the activation side, alpha = 0, and the weight
 * side, alpha = 1).  For each alphas[i] the whole smoothed W8A8 layer runs
 * on the GPU with this library's kernels -- eq. (4) from the calibration
 * peaks amax_x and the weight column peaks (computed once), the fold
 * (W * s -> INT8 and, with a LayerNorm, gamma / s, beta / s), the runtime
 * quantizer at granularity gran on the evaluation tokens x, the INT8 GEMM
 * in fp32 -- and
 *
 *   err[i] = ||y - y_ref||_F / ||y_ref||_F      (sums in fp64)
 *
 * against the caller's reference output y_ref (typically the unquantized
 * layer, f(x) W^T in fp32 or better).
 *
 *   amax_x [K] fp32 (from sq_calib_absmax, with the LayerNorm when one
 *   precedes); w [N,K] of type wt; x [M,K] of type xt; ln_gamma / ln_beta
 *   [K] fp32 or NULL (no LayerNorm: the quantizer multiplies by 1/s);
 *   y_ref [M,N] fp32; alphas: HOST array of n_alpha values in [0,1];
 *   err: DEVICE array of n_alpha doubles (out); workspace: at least
 *   sq_alpha_sweep_workspace_bytes(M,N,K) bytes of device memory, 16-byte
 *   aligned (holds every intermediate of one alpha, reused for the next).
 *   Errors as the calls it composes, SQ_ERR_WORKSPACE for a short
 *   workspace; n_alpha = 0 does nothing.
 */
size_t sq_alpha_sweep_workspace_bytes(int64_t M, int64_t N, int64_t K);
sq_status sq_alpha_sweep(const float* amax_x, const void* w, sq_dtype wt,
                         int64_t N, int64_t K, const void* x, sq_dtype xt,
                         int64_t M, const float* ln_gamma,
                         const float* ln_beta, float ln_eps,
                         const float* y_ref, const float* alphas, int n_alpha,
                         sq_act_gran gran, double* err, void* workspace,
                         size_t workspace_bytes, sq_stream stream);

/*
 * sq_sync_status -- synchronize `stream`, then return and clear the status
 * word of the current device: SQ_OK, or SQ_ERR_TIMEOUT when a kernel gave up
 * a bounded wait (its outputs are then undefined), or SQ_ERR_CUDA when the
 * synchronization itself failed.
 */
sq_status sq_sync_status(sq_stream stream);

/* Static description of a status code (never NULL). */
const char* sq_status_string(sq_status st);

/* Description of the last host-side error on the calling thread ("" if none). */
const char* sq_last_error(void);

/*
 * sq_selftest_bounded_wait -- exercises the device-side timeout path without
 * any fault: launches one CTA that waits on an mbarrier nothing arrives at,
 * with a wait limit of `limit_ns` nanoseconds (1 .. 10^9).  The wait runs out,
 * the kernel records SQ_ERR_TIMEOUT in the status word and returns normally;
 * sq_sync_status() then reports it.  Used by the fault-detection tests.
 */
sq_status sq_selftest_bounded_wait(int64_t limit_ns, sq_stream stream);

/*
 * sq_debug_bounds_enabled -- 1 if this library was built with device-side
 * bounds checks (`build.py --debug-bounds`, which writes
 * libsq_b200_debug.so), else 0.  In such a build every kernel checks each
 * global-memory offset it computes by hand (TMA copies are clipped by the
 * hardware) against its tensor's extent before the access; an offset
 * outside records SQ_ERR_BOUNDS in the status word and the access is
 * skipped -- nothing traps.  The checks cost time; the outputs are
 * otherwise those of the release build.
 */
int sq_debug_bounds_enabled(void);

/*
 * sq_selftest_bounds_check -- exercises that path without any out-of-range
 * access: one thread checks an offset equal to its tensor's extent and
 * touches no memory.  In a bounds-checked build the check records
 * SQ_ERR_BOUNDS, which sq_sync_status() then reports; otherwise nothing is
 * recorded.
 */
sq_status sq_selftest_bounds_check(sq_stream stream);

/*
 * sq_probe_mma_i8 -- measurement support (no counterpart on the pages): the
 * INT8 tensor-core rate of this GPU, the ceiling the large-M GEMM is compared
 * with.  Launches `grid` CTAs (one per SM when grid <= the SM count; each
 * takes more shared memory than two CTAs could share) that each issue
 * kblocks x 4 tcgen05.mma kind::i8 steps of 128 x 256 x 32 back to back into
 * one INT32 TMEM accumulator, from operand tiles in shared memory, with no
 * global-memory traffic.  The work is 8,388,608 * kblocks * grid int8 ops
 * (2 per multiply-add); the caller times the launch on `stream`.
 * kblocks in [1, 2^30], grid in [1, 65535], else SQ_ERR_INVALID_ARG; the
 * final wait is bounded (SQ_ERR_TIMEOUT through sq_sync_status).
 */
sq_status sq_probe_mma_i8(int64_t kblocks, int grid, sq_stream stream);

/*
 * sq_probe_mma_i8_pair -- the same measurement for the instruction form the
 * large-M GEMM uses: `pairs` clusters of two CTAs, the even CTA of each
 * issuing kblocks x 4 tcgen05.mma.cta_group::2.kind::i8 steps of
 * 256 x 256 x 32 that read A and B from both CTAs' shared memory into each
 * CTA's TMEM.  Work: 16,777,216 * kblocks * pairs int8 ops (the same per SM
 * as sq_probe_mma_i8).  kblocks in [1, 2^30], pairs in [1, 32767], else
 * SQ_ERR_INVALID_ARG; the final wait is bounded.
 */
sq_status sq_probe_mma_i8_pair(int64_t kblocks, int pairs, sq_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* SQ_H */
