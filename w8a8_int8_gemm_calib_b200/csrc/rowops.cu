// rowops.cu -- the HBM-bound steps of the smoothed W8A8 linear layer on
// sm_100a: calibration absmax (raw and LayerNorm-fused), the weight column
// peak and the smoothing factors of eq. (4), the per-output-channel weight
// quantizer, the LayerNorm fold, and the runtime fused LayerNorm + smoothing
// + INT8 activation quantizer.
//
// Sources:
//   [explainer] "SmoothQuant 如何解决激活量化难题？为什么适合 W8A8？" §三, §四
//   [review]    "SmoothQuant：大型语言模型的精准高效训练后量化 — 深度技术评审"
//               §2.2 (quantizer), §2.5-2.6 (granularity), §5.1 eq. (3),
//               §5.3 eq. (4), §5.5 (offline fold)
//   [embedded]  "嵌入式 SLM 动态权重量化：SmoothQuant 激活异常值迁移与 INT8 部署实战"
//               §二 (gamma/s, beta/s; W*diag(s); per-tensor INT8 of X_hat), §三
//
// Every fp32 operation that feeds an integer code is an explicit _rn
// intrinsic (never contracted), in the order documented in include/sq.h.
#include <cuda_runtime.h>
#include <stdint.h>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {

// ============================================================ column absmax
// X [T,K] -> out[k] = max(out[k], max_t |X[t,k]|).  A warp covers 32 chunks
// of 8 columns (256 columns: 512 B of bf16 or 1 KB of fp32 per row, fully
// coalesced 16-byte loads); the 8 warps of a CTA walk the rows of one slab,
// four rows in flight per thread.  Peaks are combined in shared memory and
// then once per column per CTA with an atomic max on the fp32 bit pattern
// (valid because every value is >= 0).
constexpr int kColWarps = 8;

template <typename T>
__global__ void __launch_bounds__(kColWarps * 32)
colmax_kernel(const T* __restrict__ x, int64_t T_, int64_t K, int64_t rows_per_slab,
              unsigned int* __restrict__ out) {
  __shared__ float part[kColWarps][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nchunk = K >> 3;
  const int64_t chunk = (int64_t)blockIdx.x * 32 + lane;
  const bool live = chunk < nchunk;
  const int64_t r0 = (int64_t)blockIdx.y * rows_per_slab;
  const int64_t r1 = min(T_, r0 + rows_per_slab);
  float m[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m[e] = 0.0f;
  if (live) {
    const T* base = x + chunk * 8;
    int64_t r = r0 + warp;
    for (; r + 3 * kColWarps < r1; r += 4 * kColWarps) {
      Raw8<T> raw[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) load_raw(base + (r + u * kColWarps) * K, raw[u]);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        float v[8];
        unpack(raw[u], v);
#pragma unroll
        for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], fabsf(v[e]));
      }
    }
    for (; r < r1; r += kColWarps) {
      Raw8<T> raw;
      load_raw(base + r * K, raw);
      float v[8];
      unpack(raw, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], fabsf(v[e]));
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[warp][lane * 8 + e] = m[e];
  __syncthreads();
  // 256 threads: one column each
  const int col = threadIdx.x;
  float v = part[0][col];
#pragma unroll
  for (int w = 1; w < kColWarps; ++w) v = fmaxf(v, part[w][col]);
  const int64_t k = (int64_t)blockIdx.x * 256 + col;
  if (k < K) atomicMax(out + k, __float_as_uint(v));
}

cudaError_t launch_colmax(const void* x, sq_dtype xt, int64_t T, int64_t K,
                          float* out, cudaStream_t st) {
  const int64_t strips = (K + 255) / 256;
  const int64_t target = (int64_t)sm_count() * 8;  // one wave of 256-thread CTAs
  int64_t slabs = (target + strips - 1) / strips;
  const int64_t min_rows = 4 * kColWarps;           // at least one unrolled step
  int64_t maxslabs = (T + min_rows - 1) / min_rows;
  if (slabs > maxslabs) slabs = maxslabs;
  if (slabs < 1) slabs = 1;
  if (slabs > 65535) slabs = 65535;
  const int64_t rows = (T + slabs - 1) / slabs;
  slabs = (T + rows - 1) / rows;
  dim3 grid((unsigned)strips, (unsigned)slabs);
  if (xt == SQ_BF16)
    colmax_kernel<uint16_t><<<grid, kColWarps * 32, 0, st>>>(
        (const uint16_t*)x, T, K, rows, (unsigned int*)out);
  else
    colmax_kernel<float><<<grid, kColWarps * 32, 0, st>>>(
        (const float*)x, T, K, rows, (unsigned int*)out);
  return cudaGetLastError();
}

// ============================================================ row kernel
// One 128-thread slice per row; 4 slices per CTA; rows are assigned to
// slices round-robin over the grid.  Slot j = 32*w + l (warp w of the slice,
// lane l) owns the 8-element chunks c = j, j+128, j+256, ... of the row.
//
// LayerNorm reduction order (the library's fixed order, shared with the
// calibration statistic): each slot accumulates its chunks in increasing c,
// elements in increasing k, from 0.0f; the 32 slots of a warp are combined
// by a butterfly (xor offsets 16, 8, 4, 2, 1: p <- p + p'); the four warp
// results as (r0 + r2) + (r1 + r3).  Mean = sum / K; variance with one fused
// multiply-add per element, (x - mean)^2 + p, in the same order, / K;
// rstd = 1 / sqrt(var + eps); y = ((x - mean) * rstd) * g + b.
//
// MAXC > 0: the thread's chunks of the row are held in registers (at most
// MAXC of them).  MAXC == 0: every pass re-reads the row (any K).
constexpr int kSlices = 4;
constexpr int kSliceThreads = 128;
constexpr size_t kColmaxSmemMax = 192 * 1024;

__device__ __forceinline__ void slice_bar(int slice) {
  asm volatile("bar.sync %0, %1;" ::"r"(slice + 1), "r"(kSliceThreads) : "memory");
}

__device__ __forceinline__ float warp_sum_butterfly(float p) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) p = __fadd_rn(p, __shfl_xor_sync(0xffffffffu, p, o));
  return p;
}
__device__ __forceinline__ float warp_max(float p) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) p = fmaxf(p, __shfl_xor_sync(0xffffffffu, p, o));
  return p;
}

template <typename T, int MAXC, bool LN, int MODE, bool COUNT>
__global__ void __launch_bounds__(kSlices * kSliceThreads)
row_kernel(RowArgs a) {
  // [slice][parity][reduction][warp]
  __shared__ float red[kSlices][2][3][4];
  extern __shared__ unsigned int colmax_s[];  // ROW_COLMAX with MAXC == 0: [K]

  const int slice = threadIdx.x / kSliceThreads;
  const int j = threadIdx.x % kSliceThreads;
  const int w = j >> 5, lane = j & 31;
  const int64_t K = a.K;
  const int64_t nchunk = K >> 3;
  const T* __restrict__ x = (const T*)a.x;
  const float* __restrict__ g = a.g;
  const float* __restrict__ b = a.b;
  const float* __restrict__ mul = a.mul;
  const float kf = (float)K;

  uint32_t dyn_smem;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_smem));
  const bool use_smem = dyn_smem > 0;
  constexpr int CM = MAXC > 0 ? MAXC : 1;
  constexpr int NCMAX = (MODE == ROW_COLMAX && MAXC > 0) ? CM * 8 : 1;
  float cmax[NCMAX];
  if constexpr (MODE == ROW_COLMAX) {
    if constexpr (MAXC > 0) {
#pragma unroll
      for (int i = 0; i < NCMAX; ++i) cmax[i] = 0.0f;
    } else {
      if (use_smem) {
        for (int64_t k = threadIdx.x; k < K; k += blockDim.x) colmax_s[k] = 0u;
        __syncthreads();
      }
    }
  }

  float static_inv = 0.0f;
  if (MODE == ROW_STATIC) static_inv = __fdiv_rn(1.0f, __ldg(a.scale));
  unsigned clipped = 0;
  int parity = 0;

  const int64_t stride = (int64_t)gridDim.x * kSlices;
  for (int64_t row = (int64_t)blockIdx.x * kSlices + slice; row < a.T; row += stride) {
    const T* xr = x + row * K;
    Raw8<T> raw[CM];
    if constexpr (MAXC > 0) {
#pragma unroll
      for (int i = 0; i < CM; ++i) {
        const int64_t c = j + (int64_t)i * kSliceThreads;
        if (c < nchunk) load_raw(xr + c * 8, raw[i]);
      }
    }
    // element access for pass p: v[8] of chunk i (MAXC>0) or chunk c (MAXC==0)
#define SQ_CHUNK_LOOP(BODY)                                                     \
    if constexpr (MAXC > 0) {                                                   \
      _Pragma("unroll") for (int i = 0; i < CM; ++i) {                          \
        const int64_t c = j + (int64_t)i * kSliceThreads;                       \
        if (c < nchunk) {                                                       \
          float v[8];                                                           \
          unpack(raw[i], v);                                                    \
          BODY                                                                  \
        }                                                                       \
      }                                                                         \
    } else {                                                                    \
      int i = 0;                                                                \
      for (int64_t c = j; c < nchunk; c += kSliceThreads, ++i) {                \
        Raw8<T> r1;                                                             \
        load_raw_cached(xr + c * 8, r1);                                        \
        float v[8];                                                             \
        unpack(r1, v);                                                          \
        BODY                                                                    \
      }                                                                         \
    }

    float mu = 0.0f, rstd = 0.0f;
    if constexpr (LN) {
      float p = 0.0f;
      SQ_CHUNK_LOOP({
        _Pragma("unroll") for (int e = 0; e < 8; ++e) p = __fadd_rn(p, v[e]);
      })
      p = warp_sum_butterfly(p);
      if (lane == 0) red[slice][parity][0][w] = p;
      slice_bar(slice);
      const float s0 = __fadd_rn(__fadd_rn(red[slice][parity][0][0], red[slice][parity][0][2]),
                                 __fadd_rn(red[slice][parity][0][1], red[slice][parity][0][3]));
      mu = __fdiv_rn(s0, kf);
      float q = 0.0f;
      SQ_CHUNK_LOOP({
        _Pragma("unroll") for (int e = 0; e < 8; ++e) {
          const float d = __fsub_rn(v[e], mu);
          q = __fmaf_rn(d, d, q);
        }
      })
      q = warp_sum_butterfly(q);
      if (lane == 0) red[slice][parity][1][w] = q;
      slice_bar(slice);
      const float s1 = __fadd_rn(__fadd_rn(red[slice][parity][1][0], red[slice][parity][1][2]),
                                 __fadd_rn(red[slice][parity][1][1], red[slice][parity][1][3]));
      const float var = __fdiv_rn(s1, kf);
      rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, a.eps)));
    }

    // y for chunk c, element e (gv/bv/mv hold the parameters of the chunk)
#define SQ_Y(e) (LN ? __fadd_rn(__fmul_rn(__fmul_rn(__fsub_rn(v[e], mu), rstd), gv[e]), bv[e]) \
                    : (mul ? __fmul_rn(v[e], mv[e]) : v[e]))
#define SQ_PARAMS                                                               \
    float gv[8], bv[8], mv[8];                                                  \
    if (LN) {                                                                   \
      load8(g + c * 8, gv);                                                     \
      if (b) load8(b + c * 8, bv); else { _Pragma("unroll") for (int e = 0; e < 8; ++e) bv[e] = 0.0f; } \
    } else if (mul) {                                                           \
      load8(mul + c * 8, mv);                                                   \
    }

    if constexpr (MODE == ROW_COLMAX) {
      SQ_CHUNK_LOOP({
        SQ_PARAMS
        _Pragma("unroll") for (int e = 0; e < 8; ++e) {
          const float y = fabsf(SQ_Y(e));
          if constexpr (MAXC > 0) {
            cmax[i * 8 + e] = fmaxf(cmax[i * 8 + e], y);
          } else if (use_smem) {
            atomicMax(&colmax_s[c * 8 + e], __float_as_uint(y));
          } else {
            atomicMax((unsigned int*)a.colmax + c * 8 + e, __float_as_uint(y));
          }
        }
      })
    } else {
      float inv = static_inv;
      if (MODE == ROW_DYNAMIC) {
        float m = 0.0f;
        SQ_CHUNK_LOOP({
          SQ_PARAMS
          _Pragma("unroll") for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(SQ_Y(e)));
        })
        m = warp_max(m);
        if (lane == 0) red[slice][parity][2][w] = m;
        slice_bar(slice);
        m = fmaxf(fmaxf(red[slice][parity][2][0], red[slice][parity][2][1]),
                  fmaxf(red[slice][parity][2][2], red[slice][parity][2][3]));
        const float delta = __fdiv_rn(fmaxf(m, 1e-7f), 127.0f);
        inv = __fdiv_rn(1.0f, delta);
        if (j == 0) a.scale[row] = delta;
      }
      int8_t* qr = a.q + row * K;
      SQ_CHUNK_LOOP({
        SQ_PARAMS
        int q[8];
        _Pragma("unroll") for (int e = 0; e < 8; ++e) q[e] = quant_code(SQ_Y(e), inv, clipped);
        uint2 pk;
        pk.x = pack4(q[0], q[1], q[2], q[3]);
        pk.y = pack4(q[4], q[5], q[6], q[7]);
        *reinterpret_cast<uint2*>(qr + c * 8) = pk;
      })
    }
#undef SQ_PARAMS
#undef SQ_Y
#undef SQ_CHUNK_LOOP
    parity ^= 1;
  }

  if constexpr (MODE == ROW_COLMAX) {
    if constexpr (MAXC > 0) {
      // slices -> global directly (each slot owns distinct columns within a slice)
#pragma unroll
      for (int i = 0; i < CM; ++i) {
        const int64_t c = j + (int64_t)i * kSliceThreads;
        if (c < nchunk) {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            atomicMax((unsigned int*)a.colmax + c * 8 + e, __float_as_uint(cmax[i * 8 + e]));
        }
      }
    } else if (use_smem) {
      __syncthreads();
      for (int64_t k = threadIdx.x; k < K; k += blockDim.x)
        atomicMax((unsigned int*)a.colmax + k, colmax_s[k]);
    }
  }
  if (COUNT && a.n_clipped) {
    // warp-aggregated count
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) clipped += __shfl_xor_sync(0xffffffffu, clipped, o);
    if (lane == 0 && clipped) atomicAdd(a.n_clipped, (unsigned long long)clipped);
  }
}

template <typename T, int MAXC, bool LN, int MODE, bool COUNT>
static cudaError_t launch_row_t(const RowArgs& a, cudaStream_t st) {
  auto kern = row_kernel<T, MAXC, LN, MODE, COUNT>;
  size_t smem = 0;
  if (MODE == ROW_COLMAX && MAXC == 0) {
    // per-CTA column peaks in shared memory when they fit; beyond that the
    // kernel updates the global peaks directly
    const size_t need = (size_t)a.K * sizeof(unsigned int);
    if (need <= kColmaxSmemMax) {
      smem = need;
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
      if (e != cudaSuccess) return e;
    }
  }
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
      &per_sm, kern, kSlices * kSliceThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int64_t want = (a.T + kSlices - 1) / kSlices;
  int64_t cap = (int64_t)sm_count() * per_sm;
  if (MODE == ROW_COLMAX) {
    // fewer, longer-lived CTAs: each flushes K column peaks at the end
    int64_t rows_each = 16;
    int64_t lim = (a.T + kSlices * rows_each - 1) / (kSlices * rows_each);
    if (want > lim) want = lim;
  }
  int64_t grid = want < cap ? want : cap;
  if (grid < 1) grid = 1;
  kern<<<(unsigned)grid, kSlices * kSliceThreads, smem, st>>>(a);
  return cudaGetLastError();
}

// Register-cached variants cover K up to 8*128*MAXC; the largest MAXC that
// compiles without spilling depends on the element type and mode (fp32 chunks
// take twice the registers of bf16 ones; the column-peak mode also keeps a
// running maximum per owned element).  Wider rows use the re-reading variant.
template <typename T, bool LN, int MODE, bool COUNT>
static cudaError_t dispatch_maxc(const RowArgs& a, cudaStream_t st) {
  constexpr bool kBf16 = sizeof(T) == 2;
  constexpr int kMax = MODE == ROW_COLMAX ? (kBf16 ? 8 : 4) : (kBf16 ? 24 : 8);
  const int64_t per_thread = (a.K / 8 + kSliceThreads - 1) / kSliceThreads;
  if (per_thread <= 1) return launch_row_t<T, 1, LN, MODE, COUNT>(a, st);
  if (per_thread <= 2) return launch_row_t<T, 2, LN, MODE, COUNT>(a, st);
  if (per_thread <= 4) return launch_row_t<T, 4, LN, MODE, COUNT>(a, st);
  if constexpr (kMax >= 8) {
    if (per_thread <= 8) return launch_row_t<T, 8, LN, MODE, COUNT>(a, st);
  }
  if constexpr (kMax >= 16) {
    if (per_thread <= 16) return launch_row_t<T, 16, LN, MODE, COUNT>(a, st);
  }
  if constexpr (kMax >= 24) {
    if (per_thread <= 24) return launch_row_t<T, 24, LN, MODE, COUNT>(a, st);
  }
  return launch_row_t<T, 0, LN, MODE, COUNT>(a, st);
}

template <typename T>
static cudaError_t dispatch_mode(const RowArgs& a, RowMode mode, cudaStream_t st) {
  const bool ln = a.g != nullptr;
  const bool cnt = a.n_clipped != nullptr;
  switch (mode) {
    case ROW_DYNAMIC:
      if (ln) return cnt ? dispatch_maxc<T, true, ROW_DYNAMIC, true>(a, st)
                         : dispatch_maxc<T, true, ROW_DYNAMIC, false>(a, st);
      return cnt ? dispatch_maxc<T, false, ROW_DYNAMIC, true>(a, st)
                 : dispatch_maxc<T, false, ROW_DYNAMIC, false>(a, st);
    case ROW_STATIC:
      if (ln) return cnt ? dispatch_maxc<T, true, ROW_STATIC, true>(a, st)
                         : dispatch_maxc<T, true, ROW_STATIC, false>(a, st);
      return cnt ? dispatch_maxc<T, false, ROW_STATIC, true>(a, st)
                 : dispatch_maxc<T, false, ROW_STATIC, false>(a, st);
    case ROW_COLMAX:
      return dispatch_maxc<T, true, ROW_COLMAX, false>(a, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_row(const RowArgs& a, sq_dtype xt, RowMode mode, cudaStream_t st) {
  if (xt == SQ_BF16) return dispatch_mode<uint16_t>(a, mode, st);
  return dispatch_mode<float>(a, mode, st);
}

// ============================================================ eq. (4)
// s_k = a^alpha / b^(1-alpha), a = amax_x[k], b = max(max_n |W[n,k]|, 1e-7)
// in fp64 (alpha = 0.5 via square roots, alpha in {0, 1} without pow), then
// one rounding to fp32, floored at 1e-4; inv_s = 1/s.  One CTA; it also
// forms the static activation step Delta(max_k a/s_k).
__global__ void __launch_bounds__(1024)
scales_kernel(const float* __restrict__ amax_x, int64_t K, float alpha,
              float* s, float* __restrict__ inv_s, float* __restrict__ delta_out) {
  __shared__ float wmax[32];
  float lmax = 0.0f;
  const double al = (double)alpha;
  for (int64_t k = threadIdx.x; k < K; k += blockDim.x) {
    const float a = amax_x[k];
    const float bw = fmaxf(s[k], 1e-7f);  // s holds the weight column peak on entry
    const double ad = (double)a, bd = (double)bw;
    double sd;
    if (alpha == 0.5f)
      sd = __ddiv_rn(__dsqrt_rn(ad), __dsqrt_rn(bd));
    else if (alpha == 1.0f)
      sd = ad;
    else if (alpha == 0.0f)
      sd = __ddiv_rn(1.0, bd);
    else
      sd = __ddiv_rn(pow(ad, al), pow(bd, __dsub_rn(1.0, al)));
    float sf = __double2float_rn(sd);
    if (!(sf >= 1e-4f)) sf = 1e-4f;
    s[k] = sf;
    inv_s[k] = __fdiv_rn(1.0f, sf);
    lmax = fmaxf(lmax, __fdiv_rn(a, sf));
  }
  if (delta_out) {
    lmax = warp_max(lmax);
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = lmax;
    __syncthreads();
    if (threadIdx.x < 32) {
      float v = threadIdx.x < (blockDim.x >> 5) ? wmax[threadIdx.x] : 0.0f;
      v = warp_max(v);
      if (threadIdx.x == 0) delta_out[0] = __fdiv_rn(fmaxf(v, 1e-7f), 127.0f);
    }
  }
}

cudaError_t launch_scales(const float* amax_x, int64_t K, float alpha, float* s,
                          float* inv_s, float* delta_out, cudaStream_t st) {
  scales_kernel<<<1, 1024, 0, st>>>(amax_x, K, alpha, s, inv_s, delta_out);
  return cudaGetLastError();
}

// ============================================================ LayerNorm fold
// gamma' = gamma / s, beta' = beta / s ([embedded] §二), fp32 division.
__global__ void fold_ln_kernel(const float* __restrict__ gamma, const float* __restrict__ beta,
                               const float* __restrict__ s, int64_t K,
                               float* __restrict__ gamma_out, float* __restrict__ beta_out) {
  for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < K;
       k += (int64_t)gridDim.x * blockDim.x) {
    const float sk = s[k];
    if (gamma_out) gamma_out[k] = __fdiv_rn(gamma[k], sk);
    if (beta_out) beta_out[k] = __fdiv_rn(beta[k], sk);
  }
}

cudaError_t launch_fold_ln(const float* gamma, const float* beta, const float* s, int64_t K,
                           float* gamma_out, float* beta_out, cudaStream_t st) {
  int64_t blocks = (K + 255) / 256;
  if (blocks > 1024) blocks = 1024;
  fold_ln_kernel<<<(unsigned)blocks, 256, 0, st>>>(gamma, beta, s, K, gamma_out, beta_out);
  return cudaGetLastError();
}

}  // namespace sq
