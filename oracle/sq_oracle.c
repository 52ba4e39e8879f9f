/*
 * sq_oracle.c -- plain, single-threaded CPU oracle of the smoothed W8A8
 * linear layer (SmoothQuant).  TEST INFRASTRUCTURE ONLY: see sq_oracle.h for
 * who may load it, the sources cited by tag, and the precision rules.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -std=c11 -shared -fPIC
 *        sq_oracle.c -lm
 * (-ffp-contract=off keeps every a*b+c as two rounded operations; the only
 * fused multiply-add is the explicit fmaf() in the variance accumulation.)
 *
 * Nothing here is blocked, vectorised or reordered: each function is the
 * definition written out as nested loops.
 */
#include "sq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* element access                                                      */
/* ------------------------------------------------------------------ */

/* bf16 -> fp32 is exact: the bf16 pattern is the upper half of the fp32 one. */
static float bf16_to_f32(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

static float load_elem(const void* p, int type, int64_t i) {
  if (type == ORC_BF16) return bf16_to_f32(((const uint16_t*)p)[i]);
  return ((const float*)p)[i];
}

/* Round to nearest, ties to even (FE_TONEAREST is the C default mode). */
static float rne(float r) { return nearbyintf(r); }

uint16_t orc_f32_to_bf16(float v) {
  uint32_t u;
  memcpy(&u, &v, sizeof u);
  if (isnan(v)) return (uint16_t)((u >> 16) | 0x0040u);
  /* add half an ulp of the bf16 result, plus one if the kept lsb is odd
   * (ties go to even), then truncate */
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------ */
/* symmetric INT8 quantizer, [review] §2.2                             */
/* ------------------------------------------------------------------ */

/* delta = max|X| / (2^(8-1) - 1).  The 1e-7 floor keeps an all-zero tensor
 * (or row) finite; it follows the small floor [embedded] §三 puts on the
 * weight peak.  An all-zero row then quantises to all zeros. */
float orc_delta(float amax) {
  float a = amax > 1e-7f ? amax : 1e-7f;
  return a / 127.0f;
}

/* X_int8 = round(X / delta), clamped to the symmetric range [-127, 127].
 * The division is taken as one fp32 reciprocal of delta followed by one fp32
 * multiply per element; round-half-to-even. */
static int8_t quant_with_inv(float v, float inv_delta, int64_t* n_clipped) {
  float r = v * inv_delta;
  if (isnan(r)) return 0;
  float q = rne(r);
  if (q > 127.0f) {
    if (n_clipped) (*n_clipped)++;
    return 127;
  }
  if (q < -127.0f) {
    if (n_clipped) (*n_clipped)++;
    return -127;
  }
  return (int8_t)q;
}

int8_t orc_quant(float v, float delta) {
  float inv = 1.0f / delta;
  return quant_with_inv(v, inv, NULL);
}

/* ------------------------------------------------------------------ */
/* LayerNorm in the canonical reduction order                          */
/* ------------------------------------------------------------------ */

#define NSLOT 128 /* 4 groups of 32 */
#define CHUNK 8

/* Sum of f(x[k]) over one row: term(k) = x[k] (sq = 0) or (x[k]-mu)^2
 * accumulated with one fused multiply-add per element (sq = 1).
 * Slot j takes the 8-wide chunks c = j, j+128, j+256, ... in increasing
 * order, elements inside a chunk in increasing order.  Each group of 32
 * slots is combined by a butterfly: five rounds, offsets 16, 8, 4, 2, 1,
 * where every slot l becomes p[l] + p[l ^ offset].  The four group results
 * are combined as (r0 + r2) + (r1 + r3). */
static float canonical_row_sum(const float* x, int64_t K, float mu, int sq) {
  float slot[NSLOT];
  for (int j = 0; j < NSLOT; ++j) slot[j] = 0.0f;
  int64_t nchunk = K / CHUNK;
  for (int64_t c = 0; c < nchunk; ++c) {
    int j = (int)(c % NSLOT);
    for (int e = 0; e < CHUNK; ++e) {
      float v = x[c * CHUNK + e];
      if (sq) {
        float d = v - mu;
        slot[j] = fmaf(d, d, slot[j]);
      } else {
        slot[j] = slot[j] + v;
      }
    }
  }
  float r[4];
  for (int g = 0; g < 4; ++g) {
    float p[32], nxt[32];
    for (int l = 0; l < 32; ++l) p[l] = slot[32 * g + l];
    for (int off = 16; off >= 1; off >>= 1) {
      for (int l = 0; l < 32; ++l) nxt[l] = p[l] + p[l ^ off];
      for (int l = 0; l < 32; ++l) p[l] = nxt[l];
    }
    r[g] = p[0];
  }
  return (r[0] + r[2]) + (r[1] + r[3]);
}

void orc_layernorm_row(const float* x, int64_t K, const float* g,
                       const float* b, float eps, float* y) {
  float kf = (float)K;
  float mu = canonical_row_sum(x, K, 0.0f, 0) / kf;
  float var = canonical_row_sum(x, K, mu, 1) / kf;
  float rstd = 1.0f / sqrtf(var + eps);
  for (int64_t k = 0; k < K; ++k) {
    float d = x[k] - mu;
    float n = d * rstd;
    float t = n * g[k];
    y[k] = t + (b ? b[k] : 0.0f);
  }
}

/* RMSNorm: the mean of squares in the same slot order (each slot's update
 * is fmaf(x, x, p)), rstd = 1 / sqrtf(ms + eps), y = (x * rstd) * g. */
void orc_rmsnorm_row(const float* x, int64_t K, const float* g, float eps,
                     float* y) {
  float kf = (float)K;
  float ms = canonical_row_sum(x, K, 0.0f, 1) / kf;
  float rstd = 1.0f / sqrtf(ms + eps);
  for (int64_t k = 0; k < K; ++k) {
    float n = x[k] * rstd;
    y[k] = n * g[k];
  }
}

/* The linear's input y of one row: the preceding norm's output, or the row
 * times inv_s (NULL: the row itself). */
static void row_output(const float* row, int64_t K, int norm, const float* g,
                       const float* b, float eps, const float* inv_s, float* y) {
  if (norm == ORC_NORM_LAYER) {
    orc_layernorm_row(row, K, g, b, eps, y);
  } else if (norm == ORC_NORM_RMS) {
    orc_rmsnorm_row(row, K, g, eps, y);
  } else {
    for (int64_t k = 0; k < K; ++k) y[k] = inv_s ? row[k] * inv_s[k] : row[k];
  }
}

/* ------------------------------------------------------------------ */
/* S1: calibration absmax ([explainer] §四; [review] §5.3 eq. (4))      */
/* ------------------------------------------------------------------ */

static void calib_absmax(const void* x, int xtype, int64_t T, int64_t K,
                         int norm, const float* gamma, const float* beta,
                         float eps, float* amax) {
  float* row = (float*)malloc(sizeof(float) * (size_t)K);
  float* y = (float*)malloc(sizeof(float) * (size_t)K);
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t k = 0; k < K; ++k) row[k] = load_elem(x, xtype, t * K + k);
    row_output(row, K, norm, gamma, beta, eps, NULL, y);
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(y[k]);
      if (a > amax[k]) amax[k] = a;
    }
  }
  free(row);
  free(y);
}

void orc_calib_absmax(const void* x, int xtype, int64_t T, int64_t K,
                      const float* gamma, const float* beta, float eps,
                      float* amax) {
  calib_absmax(x, xtype, T, K, gamma ? ORC_NORM_LAYER : ORC_NORM_NONE, gamma, beta,
               eps, amax);
}

void orc_calib_absmax_rms(const void* x, int xtype, int64_t T, int64_t K,
                          const float* gamma, float eps, float* amax) {
  calib_absmax(x, xtype, T, K, ORC_NORM_RMS, gamma, NULL, eps, amax);
}

void orc_weight_colmax(const void* w, int wtype, int64_t N, int64_t K,
                       float* amax_w) {
  for (int64_t k = 0; k < K; ++k) amax_w[k] = 0.0f;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(load_elem(w, wtype, n * K + k));
      if (a > amax_w[k]) amax_w[k] = a;
    }
}

/* ------------------------------------------------------------------ */
/* S2: smoothing factor, eq. (4) ([review] §5.3; [explainer] §三)       */
/* ------------------------------------------------------------------ */

/* s_j = max|X_j|^alpha / max|W_j|^(1-alpha), in fp64.  The weight peak is
 * floored at 1e-7 and the result at 1e-4, the guards [embedded] §三 uses.
 * alpha = 0.5 is written with square roots and alpha in {0, 1} without pow,
 * so that those three cases are correctly rounded. */
void orc_smooth_scales(const float* amax_x, const float* amax_w, int64_t K,
                       float alpha, float* s, float* inv_s) {
  double al = (double)alpha;
  for (int64_t k = 0; k < K; ++k) {
    double a = (double)amax_x[k];
    float bw = amax_w[k] > 1e-7f ? amax_w[k] : 1e-7f;
    double b = (double)bw;
    double sd;
    if (alpha == 0.5f)
      sd = sqrt(a) / sqrt(b);
    else if (alpha == 1.0f)
      sd = a;
    else if (alpha == 0.0f)
      sd = 1.0 / b;
    else
      sd = pow(a, al) / pow(b, 1.0 - al);
    float sf = (float)sd;
    if (!(sf >= 1e-4f)) sf = 1e-4f;
    s[k] = sf;
    inv_s[k] = 1.0f / sf;
  }
}

/* S3: the static activation scale is fixed from the calibration peaks of the
 * smoothed activation X_hat = X diag(s)^-1 ([review] §6.4: smoothing factors
 * and static scales come from the same calibration set; [explainer] §四). */
float orc_static_delta(const float* amax_x, const float* s, int64_t K) {
  float a = 0.0f;
  for (int64_t k = 0; k < K; ++k) {
    float v = amax_x[k] / s[k];
    if (v > a) a = v;
  }
  return orc_delta(a);
}

/* ------------------------------------------------------------------ */
/* S4: offline fold ([embedded] §二; [review] §5.1 eq. (3), §5.5)       */
/* ------------------------------------------------------------------ */

void orc_fuse_weights_q8(const void* w, int wtype, int64_t N, int64_t K,
                         const float* s, int8_t* wq, float* w_scale) {
  float* what = (float*)malloc(sizeof(float) * (size_t)K);
  for (int64_t n = 0; n < N; ++n) {
    float m = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      what[k] = load_elem(w, wtype, n * K + k) * s[k];
      float a = fabsf(what[k]);
      if (a > m) m = a;
    }
    float d = orc_delta(m);
    w_scale[n] = d;
    float inv = 1.0f / d;
    for (int64_t k = 0; k < K; ++k) wq[n * K + k] = quant_with_inv(what[k], inv, NULL);
  }
  free(what);
}

void orc_fold_into_producer(const float* s, int64_t K, float* w_scale, float* bias) {
  for (int64_t k = 0; k < K; ++k) {
    w_scale[k] = w_scale[k] / s[k];
    if (bias) bias[k] = bias[k] / s[k];
  }
}

void orc_fold_ln(const float* gamma, const float* beta, const float* s,
                 int64_t K, float* gamma_out, float* beta_out) {
  for (int64_t k = 0; k < K; ++k) {
    if (gamma && gamma_out) gamma_out[k] = gamma[k] / s[k];
    if (beta && beta_out) beta_out[k] = beta[k] / s[k];
  }
}

/* ------------------------------------------------------------------ */
/* S5: runtime activation quantizer ([embedded] §二; [review] §2.5,     */
/* §2.6, §6.3)                                                         */
/* ------------------------------------------------------------------ */

static void quant_act(const void* x, int xtype, int64_t T, int64_t K, int norm,
                      const float* gamma_s, const float* beta_s, float eps,
                      const float* inv_s, int gran, float* act_scale,
                      int8_t* xq, int64_t* n_clipped) {
  float* row = (float*)malloc(sizeof(float) * (size_t)K);
  float* y = (float*)malloc(sizeof(float) * (size_t)K);
  float static_inv = 0.0f;
  if (gran == ORC_PER_TENSOR_DYNAMIC) {
    /* first pass: the peak of |y| over every row of the call */
    float m = 0.0f;
    for (int64_t t = 0; t < T; ++t) {
      for (int64_t k = 0; k < K; ++k) row[k] = load_elem(x, xtype, t * K + k);
      row_output(row, K, norm, gamma_s, beta_s, eps, inv_s, y);
      for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(y[k]);
        if (a > m) m = a;
      }
    }
    act_scale[0] = orc_delta(m);
  }
  if (gran != ORC_PER_TOKEN_DYNAMIC) static_inv = 1.0f / act_scale[0];
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t k = 0; k < K; ++k) row[k] = load_elem(x, xtype, t * K + k);
    row_output(row, K, norm, gamma_s, beta_s, eps, inv_s, y);
    float inv;
    if (gran == ORC_PER_TOKEN_DYNAMIC) {
      float m = 0.0f;
      for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(y[k]);
        if (a > m) m = a;
      }
      float d = orc_delta(m);
      act_scale[t] = d;
      inv = 1.0f / d;
    } else {
      inv = static_inv;
    }
    for (int64_t k = 0; k < K; ++k) xq[t * K + k] = quant_with_inv(y[k], inv, n_clipped);
  }
  free(row);
  free(y);
}

void orc_quant_act(const void* x, int xtype, int64_t T, int64_t K,
                   const float* gamma_s, const float* beta_s, float eps,
                   const float* inv_s, int gran, float* act_scale,
                   int8_t* xq, int64_t* n_clipped) {
  quant_act(x, xtype, T, K, gamma_s ? ORC_NORM_LAYER : ORC_NORM_NONE, gamma_s, beta_s,
            eps, inv_s, gran, act_scale, xq, n_clipped);
}

void orc_quant_act_rms(const void* x, int xtype, int64_t T, int64_t K,
                       const float* gamma_s, float eps, int gran,
                       float* act_scale, int8_t* xq, int64_t* n_clipped) {
  quant_act(x, xtype, T, K, ORC_NORM_RMS, gamma_s, NULL, eps, NULL, gran, act_scale, xq,
            n_clipped);
}

/* ------------------------------------------------------------------ */
/* S6: INT8 GEMM with per-token x per-output-channel dequantization     */
/* ([review] §2.6 Fig. 3: scales only on the outer dimensions;          */
/* [embedded] §三 integer inner product then float rescale)             */
/* ------------------------------------------------------------------ */

void orc_gemm_w8a8(const int8_t* xq, const int8_t* wq, int64_t M, int64_t N,
                   int64_t K, const float* act_scale, int act_per_token,
                   const float* w_scale, const float* bias, const int64_t* rows,
                   int64_t nrows, float* y_f32, uint16_t* y_bf16, int32_t* acc) {
  int64_t R = rows ? nrows : M;
  for (int64_t i = 0; i < R; ++i) {
    int64_t t = rows ? rows[i] : i;
    float as = act_per_token ? act_scale[t] : act_scale[0];
    for (int64_t n = 0; n < N; ++n) {
      int64_t sum = 0;
      for (int64_t k = 0; k < K; ++k)
        sum += (int64_t)xq[t * K + k] * (int64_t)wq[n * K + k];
      int32_t a32 = (int32_t)sum; /* |sum| <= 127*127*K < 2^31 for K <= 133136 */
      float scale = as * w_scale[n];
      float y = (float)a32 * scale;
      if (bias) y = y + bias[n];
      if (acc) acc[i * N + n] = a32;
      if (y_f32) y_f32[i * N + n] = y;
      if (y_bf16) y_bf16[i * N + n] = orc_f32_to_bf16(y);
    }
  }
}
