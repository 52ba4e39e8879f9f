/*
 * sq_oracle.h -- the CPU oracle of the smoothed W8A8 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path (the
 * CUDA library under w8a8_int8_gemm_calib_b200/) never includes, links or
 * calls anything here, and this file includes nothing from it.
 *
 * Sources (cited by short tag throughout the oracle):
 *   [explainer] "SmoothQuant 如何解决激活量化难题？为什么适合 W8A8？"
 *               (offer.aigcbaba.com), sections 三 and 四.
 *   [review]    "SmoothQuant：大型语言模型的精准高效训练后量化 — 深度技术评审"
 *               (Zhongzhu's Blog), sections 2.2, 2.4-2.6, 5.1-5.5, 6.3, 6.4;
 *               eq. (3), eq. (4), Fig. 3, Fig. 6.
 *   [embedded]  "嵌入式 SLM 动态权重量化：SmoothQuant 激活异常值迁移与 INT8 部署实战"
 *               (kwkr.cn), sections 一.2, 二, 三.
 *
 * Precision: every step that decides an integer code (a quantised weight or
 * activation) is carried out in IEEE fp32, one rounding per operation, in the
 * fixed order documented beside each function, because that is the precision
 * the GPU kernels take those decisions in.  The smoothing factor of eq. (4) is
 * evaluated in fp64 and rounded once to fp32.
 *
 * Layouts: row-major, C order.  X is [T,K] (token, input channel); W is
 * [N,K] (output channel, input channel), i.e. the transpose of the review's
 * W in Y = XW, so that Y[t,n] = sum_k X[t,k] * W[n,k].
 *
 * Parity status: every function below is pinned by the "not gpu" oracle tests
 * except the fp32 rounding of eq. (4) for alpha outside {0, 0.5, 1}, where
 * libm's pow is not correctly rounded: parity unpinned beyond 1 fp32 ulp.
 */
#ifndef SQ_ORACLE_H
#define SQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Input element types accepted by the oracle.  bf16 is passed as its raw
 * 16-bit pattern and widened to fp32 exactly. */
enum { ORC_F32 = 0, ORC_BF16 = 1 };
/* Activation granularity ([review] §2.5, §2.6 Fig. 3, §6.3 O1/O3). */
enum { ORC_PER_TENSOR_STATIC = 0, ORC_PER_TOKEN_DYNAMIC = 1, ORC_PER_TENSOR_DYNAMIC = 2 };
enum { ORC_NORM_NONE = 0, ORC_NORM_LAYER = 1, ORC_NORM_RMS = 2 };

/* Quantization step of the symmetric INT8 quantizer ([review] §2.2):
 * delta = max(amax, 1e-7) / 127, in fp32. */
float orc_delta(float amax);

/* Q(v; delta): r = v * (1/delta) (one fp32 division for the reciprocal, one
 * fp32 multiply), round to nearest even, clamp to [-127, 127]; NaN -> 0. */
int8_t orc_quant(float v, float delta);

/* fp32 -> bf16 bit pattern, round to nearest even; NaN -> quiet NaN. */
uint16_t orc_f32_to_bf16(float v);

/* LayerNorm of one row in the canonical reduction order (128 slots of 8-wide
 * chunks, 5-step butterfly per 32-slot group, groups combined as
 * (r0 + r2) + (r1 + r3)).  y[k] = ((x[k] - mu) * rstd) * g[k] + b[k]. */
void orc_layernorm_row(const float* x, int64_t K, const float* g,
                       const float* b, float eps, float* y);

/* S1: running per-input-channel absmax over T calibration tokens.  If gamma
 * is non-NULL the statistic is taken of the LayerNorm output (beta may be
 * NULL = 0).  amax[K] is read and updated in place. */
void orc_calib_absmax(const void* x, int xtype, int64_t T, int64_t K,
                      const float* gamma, const float* beta, float eps,
                      float* amax);

/* Per-input-channel absmax of the weights: amax_w[k] = max_n |W[n,k]|. */
void orc_weight_colmax(const void* w, int wtype, int64_t N, int64_t K,
                       float* amax_w);

/* S2: smoothing factors of eq. (4) ([review] §5.3), in fp64, then
 * s = max((float)s64, 1e-4f) and inv_s = 1/s in fp32. */
void orc_smooth_scales(const float* amax_x, const float* amax_w, int64_t K,
                       float alpha, float* s, float* inv_s);

/* S3: static per-tensor activation step delta_A = delta(max_k amax_x[k]/s[k]). */
float orc_static_delta(const float* amax_x, const float* s, int64_t K);

/* S4: W_hat = W * s (per input channel); per-output-channel symmetric INT8. */
void orc_fuse_weights_q8(const void* w, int wtype, int64_t N, int64_t K,
                         const float* s, int8_t* wq, float* w_scale);

/* RMSNorm (the norm of models without a LayerNorm mean or beta): the mean
 * of squares in the LayerNorm's slot order, each slot updated by
 * fmaf(x, x, p); ms = sum / K; rstd = 1 / sqrtf(ms + eps);
 * y = (x * rstd) * g.  Its smoothing fold is g' = g / s (no beta). */
void orc_rmsnorm_row(const float* x, int64_t K, const float* g, float eps,
                     float* y);

/* S1 through an RMSNorm with the original gamma. */
void orc_calib_absmax_rms(const void* x, int xtype, int64_t T, int64_t K,
                          const float* gamma, float eps, float* amax);

/* S5 with y = RMSNorm'(x) (gamma_s = gamma / s); granularities as
 * orc_quant_act. */
void orc_quant_act_rms(const void* x, int xtype, int64_t T, int64_t K,
                       const float* gamma_s, float eps, int gran,
                       float* act_scale, int8_t* xq, int64_t* n_clipped);

/* The fold into a producing linear ([review] §5.5: s folds into the
 * previous layer's parameters): the producer's output channel k feeds the
 * consumer's input channel k, so its per-output-channel scale and bias are
 * divided by s_k (one fp32 division each): w_scale[k] /= s[k],
 * bias[k] /= s[k] (bias may be NULL).  With s > 0 a ReLU between the two
 * commutes with the division. */
void orc_fold_into_producer(const float* s, int64_t K, float* w_scale, float* bias);

/* S4: LayerNorm fold gamma' = gamma / s, beta' = beta / s ([embedded] §二). */
void orc_fold_ln(const float* gamma, const float* beta, const float* s,
                 int64_t K, float* gamma_out, float* beta_out);

/* S5: runtime activation quantizer.  y = LN'(x) with (gamma_s, beta_s) when
 * gamma_s != NULL, else y = x * inv_s (inv_s NULL = 1).  Per-token: writes
 * act_scale[t] = delta(max_k |y[t,k]|).  Static: reads act_scale[0].
 * Per-tensor dynamic (the review's SmoothQuant-O2, §6.3; dynamic steps §2.5):
 * writes act_scale[0] = delta(max_{t,k} |y[t,k]|) over the whole call, then
 * quantizes every row with it.  Peaks skip NaN (a NaN is never > m).
 * n_clipped (may be NULL) is incremented by the number of elements whose
 * rounded code fell outside [-127, 127] and was saturated. */
void orc_quant_act(const void* x, int xtype, int64_t T, int64_t K,
                   const float* gamma_s, const float* beta_s, float eps,
                   const float* inv_s, int gran, float* act_scale,
                   int8_t* xq, int64_t* n_clipped);

/* S6: acc[t,n] = sum_k xq[t,k]*wq[n,k] (int32, exact);
 * y = (float)acc * (act_scale[t or 0] * w_scale[n]), then + bias[n] when
 * bias != NULL (one more fp32 addition: the linear's bias is untouched by
 * the smoothing, [review] §5.1 eq. (3)).  Only the rows listed in
 * rows[0..nrows) are computed (rows == NULL: all M rows, nrows ignored);
 * output row i of y/acc corresponds to input row rows[i].  y_bf16 and acc
 * may be NULL; y_f32 may be NULL. */
void orc_gemm_w8a8(const int8_t* xq, const int8_t* wq, int64_t M, int64_t N,
                   int64_t K, const float* act_scale, int act_per_token,
                   const float* w_scale, const float* bias, const int64_t* rows,
                   int64_t nrows, float* y_f32, uint16_t* y_bf16, int32_t* acc);

#ifdef __cplusplus
}
#endif
#endif
