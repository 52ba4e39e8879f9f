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

#include <mutex>

#include "launch.cuh"
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

template <typename T>
__global__ void __launch_bounds__(kColWarps * 32)
colmax_kernel(const T* __restrict__ x, int64_t T_, int64_t K, int64_t rows_per_slab,
              unsigned int* __restrict__ out, unsigned int* status) {
  __shared__ float part[kColWarps][256];
  pdl_launch_dependents();
  pdl_wait();
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
    constexpr int U = sizeof(T) == 2 ? 8 : 4;  // 128 B in flight per thread
    for (; r + (U - 1) * kColWarps < r1; r += U * kColWarps) {
      Raw8<T> raw[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        raw[u] = Raw8<T>{};
        if (in_bounds(chunk * 8 + (r + u * kColWarps) * K, 8, T_ * K, status))
          load_raw(base + (r + u * kColWarps) * K, raw[u]);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float v[8];
        unpack(raw[u], v);
#pragma unroll
        for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], fabsf(v[e]));
      }
    }
    for (; r < r1; r += kColWarps) {
      Raw8<T> raw{};
      if (in_bounds(chunk * 8 + r * K, 8, T_ * K, status)) load_raw(base + r * K, raw);
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
  if (k < K && in_bounds(k, 1, K, status)) atomicMax(out + k, __float_as_uint(v));
}

// Slabs of rows per column strip so that the grid is one wave of resident
// CTAs (per_sm of them on every SM): a second, partial wave would leave a
// few CTAs streaming alone at the end, far below the HBM rate (65536 x 8192
// bf16 peaks: 262 us with 768 CTAs on 740 slots).
int64_t strip_rows(int64_t T, int64_t strips, int per_sm) {
  const int64_t target = (int64_t)sm_count() * per_sm;
  int64_t slabs = target / strips;
  if (slabs < 1) slabs = 1;
  const int64_t min_rows = 8 * kColWarps;  // at least one unrolled step
  const int64_t maxslabs = (T + min_rows - 1) / min_rows;
  if (slabs > maxslabs) slabs = maxslabs;
  if (slabs > 65535) slabs = 65535;
  if (slabs < 1) slabs = 1;
  return (T + slabs - 1) / slabs;
}

// Resident CTAs per SM of a kernel at kColWarps warps (queried once per
// device and instantiation).
template <typename Kern>
int strip_occupancy(Kern kern, std::once_flag* once, int* occ) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 1;
  std::call_once(once[dev], [&] {
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kColWarps * 32, 0);
    occ[dev] = n < 1 ? 1 : n;
  });
  return occ[dev];
}

// Column strips stream the rows with plain 16-byte loads and no
// synchronisation at all; measured faster here than staging whole rows
// through the shared-memory ring, where every row waits for all the warps
// that share it before its slot is refilled (W of 12288 x 4096 bf16: 30.8 us
// against 55 us).
cudaError_t launch_colmax(const void* x, sq_dtype xt, int64_t T, int64_t K, float* out,
                          cudaStream_t st) {
  const int64_t strips = (K + 255) / 256;
  static std::once_flag once[2][64];
  static int occ[2][64];
  const int per_sm = xt == SQ_BF16 ? strip_occupancy(colmax_kernel<uint16_t>, once[0], occ[0])
                                   : strip_occupancy(colmax_kernel<float>, once[1], occ[1]);
  const int64_t rows = strip_rows(T, strips, per_sm);
  dim3 grid((unsigned)strips, (unsigned)((T + rows - 1) / rows));
  if (xt == SQ_BF16)
    return launch_pdl(colmax_kernel<uint16_t>, grid, dim3(kColWarps * 32), 0, st,
                      (const uint16_t*)x, T, K, rows, (unsigned int*)out, status_word());
  return launch_pdl(colmax_kernel<float>, grid, dim3(kColWarps * 32), 0, st, (const float*)x, T,
                    K, rows, (unsigned int*)out, status_word());
}

// ============================================================ strip quantizer
// The activation quantizer when no LayerNorm precedes and the step is one
// number for the whole call: y = x * m[k] (or x) and Q(y; Delta) are
// independent per element, so the call is a plain stream -- the column-strip
// layout of colmax_kernel (a warp per 256 columns and 8 rows, several rows
// in flight per thread), each lane's 8 multipliers in registers, 8 codes
// stored per lane per row.  PEAK: no codes; the peak of |y| over the call
// (NaN skipped) is folded into *peak with one atomic max per warp (the first
// pass of per-tensor dynamic quantization).
template <typename T, bool PEAK>
__global__ void __launch_bounds__(kColWarps * 32)
strip_quant_kernel(const T* __restrict__ x, int64_t T_, int64_t K, int64_t rows_per_slab,
                   const float* __restrict__ mul, const float* scale, int8_t* __restrict__ q,
                   unsigned long long* n_clipped, unsigned int* peak, unsigned int* status) {
  pdl_launch_dependents();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nchunk = K >> 3;
  const int64_t chunk = (int64_t)blockIdx.x * 32 + lane;
  const bool live = chunk < nchunk;
  const int64_t r0 = (int64_t)blockIdx.y * rows_per_slab;
  const int64_t r1 = min(T_, r0 + rows_per_slab);
  float m8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m8[e] = 1.0f;
  if (live && mul) load8(mul + chunk * 8, m8);
  const float inv = PEAK ? 0.0f : __fdiv_rn(1.0f, __ldcg(scale));
  const bool count = n_clipped != nullptr;
  unsigned clipped = 0;
  float pk = 0.0f;
  auto work = [&](const Raw8<T>& raw, int64_t r) {
    float v[8];
    unpack(raw, v);
    if (mul) {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = __fmul_rn(v[e], m8[e]);
    }
    if constexpr (PEAK) {
#pragma unroll
      for (int e = 0; e < 8; ++e) pk = fmaxf(pk, fabsf(v[e]));
    } else {
      uint32_t b[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) b[e] = qbits(v[e], inv, count, clipped);
      if (in_bounds(r * K + chunk * 8, 8, T_ * K, status)) store_codes(q + r * K + chunk * 8, b);
    }
  };
  if (live) {
    const T* base = x + chunk * 8;
    constexpr int U = sizeof(T) == 2 ? 8 : 4;  // 128 B in flight per thread
    int64_t r = r0 + warp;
    for (; r + (U - 1) * kColWarps < r1; r += U * kColWarps) {
      Raw8<T> raw[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        raw[u] = Raw8<T>{};
        if (in_bounds(chunk * 8 + (r + u * kColWarps) * K, 8, T_ * K, status))
          load_raw(base + (r + u * kColWarps) * K, raw[u]);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) work(raw[u], r + u * kColWarps);
    }
    for (; r < r1; r += kColWarps) {
      Raw8<T> raw{};
      if (in_bounds(chunk * 8 + r * K, 8, T_ * K, status)) load_raw(base + r * K, raw);
      work(raw, r);
    }
  }
  if constexpr (PEAK) {
    pk = warp_max(pk);
    if (lane == 0) atomicMax(peak, __float_as_uint(pk));
  } else if (count) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) clipped += __shfl_xor_sync(0xffffffffu, clipped, o);
    if (lane == 0 && clipped) atomicAdd(n_clipped, (unsigned long long)clipped);
  }
}

template <typename T, bool PEAK>
cudaError_t launch_strip_quant_t(const RowArgs& a, cudaStream_t st) {
  static std::once_flag once[64];
  static int occ[64];
  const int per_sm = strip_occupancy(strip_quant_kernel<T, PEAK>, once, occ);
  const int64_t strips = (a.K + 255) / 256;
  const int64_t rows = strip_rows(a.T, strips, per_sm);
  dim3 grid((unsigned)strips, (unsigned)((a.T + rows - 1) / rows));
  return launch_pdl(strip_quant_kernel<T, PEAK>, grid, dim3(kColWarps * 32), 0, st,
                    (const T*)a.x, a.T, a.K, rows, a.mul, (const float*)a.scale, a.q,
                    a.n_clipped, reinterpret_cast<unsigned int*>(a.peak), status_word());
}

cudaError_t launch_strip_quant(const RowArgs& a, sq_dtype xt, RowMode mode, cudaStream_t st) {
  if (mode == ROW_PEAK)
    return xt == SQ_BF16 ? launch_strip_quant_t<uint16_t, true>(a, st)
                         : launch_strip_quant_t<float, true>(a, st);
  return xt == SQ_BF16 ? launch_strip_quant_t<uint16_t, false>(a, st)
                       : launch_strip_quant_t<float, false>(a, st);
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
// MAXC > 0: the thread's chunks of a row are held in registers (at most MAXC
// of them) and the next row's chunks are loaded while the current row is
// processed.  MAXC == 0: every pass re-reads the row (any K).  PREG: the
// thread's per-column parameters (gamma/beta, or the multiplier) stay in
// registers for all its rows.
constexpr int kSlices = 4;
constexpr int kSliceThreads = 128;
constexpr size_t kColmaxSmemMax = 192 * 1024;

__device__ __forceinline__ void slice_bar(int slice) {
  asm volatile("bar.sync %0, %1;" ::"r"(slice + 1), "r"(kSliceThreads) : "memory");
}


// Calls f(i, c, v[8]) for every chunk the thread owns, in increasing c.
template <int MAXC, typename T, typename F>
__device__ __forceinline__ void for_chunks(const Raw8<T> (&raw)[MAXC > 0 ? MAXC : 1],
                                           const T* xr, int j, int64_t nchunk, F&& f,
                                           int64_t row_off = 0, int64_t size = 0,
                                           unsigned int* status = nullptr) {
  if constexpr (MAXC > 0) {
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
      const int64_t c = j + (int64_t)i * kSliceThreads;
      if (c < nchunk) {
        float v[8];
        unpack(raw[i], v);
        f(i, c, v);
      }
    }
  } else {
    int i = 0;
    for (int64_t c = j; c < nchunk; c += kSliceThreads, ++i) {
      Raw8<T> r{};
      if (in_bounds(row_off + c * 8, 8, size, status)) load_raw_cached(xr + c * 8, r);
      float v[8];
      unpack(r, v);
      f(i, c, v);
    }
  }
}

template <int MAXC, typename T>
__device__ __forceinline__ void load_row(Raw8<T> (&raw)[MAXC > 0 ? MAXC : 1], const T* xr, int j,
                                         int64_t nchunk) {
  if constexpr (MAXC > 0) {
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
      const int64_t c = j + (int64_t)i * kSliceThreads;
      if (c < nchunk) load_raw(xr + c * 8, raw[i]);
    }
  }
}

template <typename T, int MAXC, bool LN, int MODE, bool COUNT, bool PREG, bool PF>
__global__ void __launch_bounds__(kSlices * kSliceThreads)
row_kernel(RowArgs a) {
  // [slice][parity][reduction][warp]
  __shared__ float red[kSlices][2][3][4];
  extern __shared__ unsigned int colmax_s[];  // ROW_COLMAX: per-CTA column peaks [K]
  pdl_launch_dependents();
  pdl_wait();
  if constexpr (!LN)
    fold_columns(a.mul, a.fold_g, a.fold_b, a.fold_g_out, a.fold_b_out, a.K, threadIdx.x,
                 blockDim.x);

  uint32_t dyn_smem;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_smem));
  const bool use_smem = dyn_smem > 0;
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

  constexpr int CM = MAXC > 0 ? MAXC : 1;
  constexpr int NCMAX = (MODE == ROW_COLMAX && MAXC > 0) ? CM * 8 : 1;
  constexpr int NP = PREG ? CM * 8 : 1;
  float cmax[NCMAX];
#pragma unroll
  for (int i = 0; i < NCMAX; ++i) cmax[i] = 0.0f;
  if constexpr (MODE == ROW_COLMAX) {
    if (use_smem) {
      for (int64_t k = threadIdx.x; k < K; k += blockDim.x) colmax_s[k] = 0u;
      __syncthreads();
    }
  }

  // per-column parameters: LN gamma/beta, or the column multiplier
  float pg[NP], pb[NP];
  if constexpr (PREG) {
#pragma unroll
    for (int i = 0; i < CM; ++i) {
      const int64_t c = j + (int64_t)i * kSliceThreads;
      float t0[8], t1[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) { t0[e] = 1.0f; t1[e] = 0.0f; }
      if (c < nchunk) {
        if (LN) {
          load8(g + c * 8, t0);
          if (b) load8(b + c * 8, t1);
        } else if (mul) {
          load8(mul + c * 8, t0);
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) { pg[i * 8 + e] = t0[e]; pb[i * 8 + e] = t1[e]; }
    }
  }
  // parameters of chunk (i, c) into g8/b8
  auto params = [&](int i, int64_t c, float (&g8)[8], float (&b8)[8]) {
    if constexpr (PREG) {
#pragma unroll
      for (int e = 0; e < 8; ++e) { g8[e] = pg[i * 8 + e]; b8[e] = pb[i * 8 + e]; }
    } else {
      if (LN) {
        load8(g + c * 8, g8);
        if (b) load8(b + c * 8, b8);
        else {
#pragma unroll
          for (int e = 0; e < 8; ++e) b8[e] = 0.0f;
        }
      } else if (mul) {
        load8(mul + c * 8, g8);
      }
    }
  };

  float static_inv = 0.0f;
  if (MODE == ROW_STATIC) static_inv = __fdiv_rn(1.0f, __ldcg(a.scale));
  unsigned clipped = 0;
  int parity = 0;
  float peak = 0.0f;  // ROW_PEAK: this thread's running max of |y| (NaN skipped)

  const int64_t stride = (int64_t)gridDim.x * kSlices;
  int64_t row = (int64_t)blockIdx.x * kSlices + slice;
  Raw8<T> cur[CM];
  if (row < a.T && in_bounds(row * K, K, a.T * K, a.status))
    load_row<MAXC>(cur, x + row * K, j, nchunk);
  while (row < a.T) {
    const int64_t nrow = row + stride;
    Raw8<T> nxt[PF ? CM : 1];
    if constexpr (PF) {
      if (nrow < a.T && in_bounds(nrow * K, K, a.T * K, a.status))
        load_row<MAXC>(nxt, x + nrow * K, j, nchunk);
    }
    const T* xr = x + row * K;
    // the thread's chunks of this row (re-read from global memory when they
    // are not held in registers, the row's extent checked in debug builds)
    auto chunks = [&](auto&& f) { for_chunks<MAXC>(cur, xr, j, nchunk, f, row * K, a.T * K, a.status); };

    float mu = 0.0f, rstd = 0.0f;
    if constexpr (LN) {
      if (!a.rms) {  // RMSNorm: no mean (mu = 0, beta NULL)
        float p = 0.0f;
        chunks([&](int, int64_t, const float (&v)[8]) {
#pragma unroll
          for (int e = 0; e < 8; ++e) p = __fadd_rn(p, v[e]);
        });
        p = warp_sum_butterfly(p);
        if (lane == 0) red[slice][parity][0][w] = p;
        slice_bar(slice);
        const float s0 = __fadd_rn(__fadd_rn(red[slice][parity][0][0], red[slice][parity][0][2]),
                                   __fadd_rn(red[slice][parity][0][1], red[slice][parity][0][3]));
        mu = __fdiv_rn(s0, kf);
      }
      float q = 0.0f;
      chunks([&](int, int64_t, const float (&v)[8]) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float d = __fsub_rn(v[e], mu);
          q = __fmaf_rn(d, d, q);
        }
      });
      q = warp_sum_butterfly(q);
      if (lane == 0) red[slice][parity][1][w] = q;
      slice_bar(slice);
      const float s1 = __fadd_rn(__fadd_rn(red[slice][parity][1][0], red[slice][parity][1][2]),
                                 __fadd_rn(red[slice][parity][1][1], red[slice][parity][1][3]));
      const float var = __fdiv_rn(s1, kf);
      rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, a.eps)));
    }
    // y of element e given the chunk's parameters
    auto yv = [&](float v, float gq, float bq) -> float {
      if constexpr (LN) {
        return __fadd_rn(__fmul_rn(__fmul_rn(__fsub_rn(v, mu), rstd), gq), bq);
      } else {
        return mul ? __fmul_rn(v, gq) : v;
      }
    };

    if constexpr (MODE == ROW_COLMAX) {
      chunks([&](int i, int64_t c, const float (&v)[8]) {
        float g8[8], b8[8];
        params(i, c, g8, b8);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float y = fabsf(yv(v[e], g8[e], b8[e]));
          if constexpr (MAXC > 0) {
            cmax[i * 8 + e] = fmaxf(cmax[i * 8 + e], y);
          } else {
            if (use_smem) atomicMax(&colmax_s[c * 8 + e], peak_bits(y));
            else if (in_bounds(c * 8 + e, 1, K, a.status))
              atomicMax((unsigned int*)a.colmax + c * 8 + e, peak_bits(y));
          }
        }
      });
    } else if constexpr (MODE == ROW_PEAK) {
      chunks([&](int i, int64_t c, const float (&v)[8]) {
        float g8[8], b8[8];
        params(i, c, g8, b8);
#pragma unroll
        for (int e = 0; e < 8; ++e) peak = fmaxf(peak, fabsf(yv(v[e], g8[e], b8[e])));
      });
    } else {
      float inv = static_inv;
      if constexpr (MODE == ROW_DYNAMIC) {
        float m = 0.0f;
        chunks([&](int i, int64_t c, const float (&v)[8]) {
          float g8[8], b8[8];
          params(i, c, g8, b8);
#pragma unroll
          for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(yv(v[e], g8[e], b8[e])));
        });
        m = warp_max(m);
        if (lane == 0) red[slice][parity][2][w] = m;
        slice_bar(slice);
        m = fmaxf(fmaxf(red[slice][parity][2][0], red[slice][parity][2][1]),
                  fmaxf(red[slice][parity][2][2], red[slice][parity][2][3]));
        const float delta = __fdiv_rn(fmaxf(m, 1e-7f), 127.0f);
        inv = __fdiv_rn(1.0f, delta);
        if (j == 0 && in_bounds(row, 1, a.T, a.status)) a.scale[row] = delta;
      }
      int8_t* qr = a.q + row * K;
      chunks([&](int i, int64_t c, const float (&v)[8]) {
        float g8[8], b8[8];
        params(i, c, g8, b8);
        int q[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) q[e] = quant_code(yv(v[e], g8[e], b8[e]), inv, clipped);
        uint2 pk;
        pk.x = pack4(q[0], q[1], q[2], q[3]);
        pk.y = pack4(q[4], q[5], q[6], q[7]);
        if (in_bounds(row * K + c * 8, 8, a.T * K, a.status))
          *reinterpret_cast<uint2*>(qr + c * 8) = pk;
      });
    }
    parity ^= 1;
    row = nrow;
    if constexpr (MAXC > 0) {
      if constexpr (PF) {
#pragma unroll
        for (int i = 0; i < CM; ++i) cur[i] = nxt[i];
      } else {
        if (row < a.T && in_bounds(row * K, K, a.T * K, a.status))
          load_row<MAXC>(cur, x + row * K, j, nchunk);
      }
    }
  }

  if constexpr (MODE == ROW_COLMAX) {
    if constexpr (MAXC > 0) {
      // the four slices own the same columns: combine them in shared memory
#pragma unroll
      for (int i = 0; i < CM; ++i) {
        const int64_t c = j + (int64_t)i * kSliceThreads;
        if (c < nchunk) {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            atomicMax(&colmax_s[c * 8 + e], __float_as_uint(cmax[i * 8 + e]));
        }
      }
    }
    if (use_smem) {
      __syncthreads();
      for (int64_t k = threadIdx.x; k < K; k += blockDim.x)
        if (in_bounds(k, 1, K, a.status)) atomicMax((unsigned int*)a.colmax + k, colmax_s[k]);
    }
  }
  if constexpr (MODE == ROW_PEAK) {
    peak = warp_max(peak);
    if (lane == 0) atomicMax(reinterpret_cast<unsigned int*>(a.peak), __float_as_uint(peak));
  }
  if (COUNT && a.n_clipped) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) clipped += __shfl_xor_sync(0xffffffffu, clipped, o);
    if (lane == 0 && clipped) atomicAdd(a.n_clipped, (unsigned long long)clipped);
  }
}

template <typename T, int MAXC, bool LN, int MODE, bool COUNT>
static cudaError_t launch_row_t(const RowArgs& a, cudaStream_t st) {
  constexpr bool kBf16 = sizeof(T) == 2;
  constexpr bool PF = MAXC > 0 && MAXC <= (kBf16 ? (MODE == ROW_COLMAX ? 4 : 8) : 2);
  constexpr bool PREG = MAXC > 0 && MAXC <= 4 && MODE != ROW_COLMAX;
  auto kern = row_kernel<T, MAXC, LN, MODE, COUNT, PREG, PF>;
  size_t smem = 0;
  if (MODE == ROW_COLMAX && (size_t)a.K * sizeof(unsigned int) <= kColmaxSmemMax)
    smem = (size_t)a.K * sizeof(unsigned int);
  // attribute and occupancy are queried once per instantiation and device
  // (at the largest shared-memory size this variant ever uses)
  static std::once_flag once[64];
  static cudaError_t init_err[64];
  static int per_sm_cache[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) return e != cudaSuccess ? e : cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] {
    const size_t top = MODE == ROW_COLMAX ? kColmaxSmemMax : 0;
    cudaError_t r = cudaSuccess;
    if (top) r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)top);
    int n = 0;
    if (r == cudaSuccess)
      r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, kSlices * kSliceThreads, top);
    per_sm_cache[dev] = n < 1 ? 1 : n;
    init_err[dev] = r;
  });
  if (init_err[dev] != cudaSuccess) return init_err[dev];
  int per_sm = per_sm_cache[dev];
  // column peaks are flushed once per CTA: one CTA per SM
  if (MODE == ROW_COLMAX) per_sm = 1;
  int64_t want = (a.T + kSlices - 1) / kSlices;
  int64_t cap = (int64_t)sm_count() * per_sm;
  int64_t grid = want < cap ? want : cap;
  if (grid < 1) grid = 1;
  return launch_pdl(kern, dim3((unsigned)grid), dim3(kSlices * kSliceThreads), smem, st, a);
}

// Rows too wide for the shared-memory pipeline (rowpipe.cu) take the
// re-reading variant, which serves any K.
template <typename T, bool LN, int MODE, bool COUNT>
static cudaError_t dispatch_maxc(const RowArgs& a, cudaStream_t st) {
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
    case ROW_PEAK:
      return ln ? dispatch_maxc<T, true, ROW_PEAK, false>(a, st)
                : dispatch_maxc<T, false, ROW_PEAK, false>(a, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_row(const RowArgs& args, sq_dtype xt, RowMode mode, cudaStream_t st) {
  RowArgs a = args;
  a.status = status_word();
  // static steps on bf16 rows without a LayerNorm: whole rows in registers
  if (rowreg_fits(a.K, xt, mode, a.g != nullptr)) return launch_rowreg(a, mode, st);
  // no LayerNorm and one step for the whole call: a plain element stream
  const bool folds = a.fold_g_out || a.fold_b_out;
  if (!a.g && !folds && (mode == ROW_STATIC || mode == ROW_PEAK))
    return launch_strip_quant(a, xt, mode, st);
  if (rowpipe_fits(a.K, xt, mode, a.g != nullptr))
    return launch_rowpipe(a, xt, mode, st);
  if (xt == SQ_BF16) return dispatch_mode<uint16_t>(a, mode, st);
  return dispatch_mode<float>(a, mode, st);
}

// ============================================================ eq. (4)
// s_k = a^alpha / b^(1-alpha), a = amax_x[k], b = max(max_n |W[n,k]|, 1e-7)
// in fp64 (alpha = 0.5 via square roots, alpha in {0, 1} without pow), then
// one rounding to fp32, floored at 1e-4; inv_s = 1/s.  Each CTA also forms
// Delta(max over its channels of a/s_k) and raises delta_out to it with an
// atomic max on the (non-negative) fp32 bits: Delta is non-decreasing in its
// argument, so the maximum over CTAs is Delta of the maximum over channels.
constexpr int kScaleThreads = 256;

__global__ void __launch_bounds__(kScaleThreads)
scales_kernel(const float* __restrict__ amax_x, const float* amax_w, int64_t K, float alpha,
              float* s, float* __restrict__ inv_s, unsigned int* __restrict__ delta_out) {
  __shared__ float wmax[kScaleThreads / 32];
  pdl_launch_dependents();
  pdl_wait();
  float lmax = 0.0f;
  const double al = (double)alpha;
  for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < K;
       k += (int64_t)gridDim.x * blockDim.x) {
    const float a = amax_x[k];
    const float bw = fmaxf(amax_w[k], 1e-7f);  // amax_w may be s itself (read before written)
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
      if (threadIdx.x == 0)
        atomicMax(delta_out, __float_as_uint(__fdiv_rn(fmaxf(v, 1e-7f), 127.0f)));
    }
  }
}

cudaError_t launch_scales(const float* amax_x, const float* amax_w, int64_t K, float alpha,
                          float* s, float* inv_s, float* delta_out, cudaStream_t st) {
  if (delta_out) {
    cudaError_t e = cudaMemsetAsync(delta_out, 0, sizeof(float), st);
    if (e != cudaSuccess) return e;
  }
  int64_t blocks = (K + kScaleThreads - 1) / kScaleThreads;
  if (blocks > 4 * (int64_t)sm_count()) blocks = 4 * (int64_t)sm_count();
  return launch_pdl(scales_kernel, dim3((unsigned)blocks), dim3(kScaleThreads), 0, st, amax_x,
                    amax_w, K, alpha, s, inv_s, (unsigned int*)delta_out);
}

// ============================================================ zero fill
__global__ void __launch_bounds__(256) zero_kernel(uint32_t* p, int64_t n) {
  pdl_launch_dependents();
  pdl_wait();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    p[i] = 0u;
}

cudaError_t launch_zero(void* p, size_t bytes, cudaStream_t st) {
  if (bytes % 4 != 0) return cudaErrorInvalidValue;
  const int64_t n = (int64_t)(bytes / 4);
  if (n == 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 4 * (int64_t)sm_count()) blocks = 4 * (int64_t)sm_count();
  return launch_pdl(zero_kernel, dim3((unsigned)blocks), dim3(256), 0, st, (uint32_t*)p, n);
}

// ============================================================ per-tensor step
// The second step of per-tensor dynamic quantization: the peak folded into
// act_scale[0] by the ROW_PEAK pass becomes Delta = max(peak, 1e-7) / 127.
__global__ void peak_to_delta_kernel(float* act_scale) {
  pdl_launch_dependents();
  pdl_wait();
  if (threadIdx.x == 0) act_scale[0] = __fdiv_rn(fmaxf(act_scale[0], 1e-7f), 127.0f);
}

cudaError_t launch_peak_to_delta(float* act_scale, cudaStream_t st) {
  return launch_pdl(peak_to_delta_kernel, dim3(1), dim3(32), 0, st, act_scale);
}

// ============================================================ output error
// sum (y - r)^2 and sum r^2 in fp64, deterministic: each thread accumulates
// a grid-stride share, warps and blocks reduce, each block writes its two
// partial sums to its own slot, and one block adds the slots in a fixed
// order (a strided share per thread, then a halving tree).
constexpr int kErrThreads = 256;

int output_error_blocks(int64_t n) {
  int64_t blocks = (n + kErrThreads - 1) / kErrThreads;
  const int64_t cap = 8 * (int64_t)sm_count();
  if (blocks > cap) blocks = cap;
  return blocks < 1 ? 1 : (int)blocks;
}

size_t output_error_scratch_bytes() { return 2 * sizeof(double) * 8 * (size_t)sm_count(); }

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(kErrThreads)
output_error_kernel(const float* __restrict__ y, const float* __restrict__ r, int64_t n,
                    double* part_out) {
  __shared__ double part[2][kErrThreads / 32];
  pdl_launch_dependents();
  pdl_wait();
  double num = 0.0, den = 0.0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const double a = (double)__ldcg(y + i), b = (double)__ldcg(r + i);
    const double d = a - b;
    num += d * d;
    den += b * b;
  }
  num = warp_sum_d(num);
  den = warp_sum_d(den);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    part[0][warp] = num;
    part[1][warp] = den;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double a = 0.0, b = 0.0;
    for (int w = 0; w < kErrThreads / 32; ++w) {
      a += part[0][w];
      b += part[1][w];
    }
    part_out[2 * blockIdx.x] = a;
    part_out[2 * blockIdx.x + 1] = b;
  }
}

// One block of kErrThreads: the slots are read in parallel (a single thread
// walking them would wait out one memory latency after another).
__global__ void __launch_bounds__(kErrThreads)
output_error_final_kernel(const double* part, int nblocks, double* err) {
  __shared__ double s[2][kErrThreads];
  pdl_launch_dependents();
  pdl_wait();
  const int t = threadIdx.x;
  double num = 0.0, den = 0.0;
  for (int i = t; i < nblocks; i += kErrThreads) {
    num += part[2 * i];
    den += part[2 * i + 1];
  }
  s[0][t] = num;
  s[1][t] = den;
  __syncthreads();
  for (int h = kErrThreads / 2; h > 0; h >>= 1) {
    if (t < h) {
      s[0][t] += s[0][t + h];
      s[1][t] += s[1][t + h];
    }
    __syncthreads();
  }
  if (t == 0) {
    num = s[0][0];
    den = s[1][0];
    *err = den > 0.0 ? sqrt(num / den) : (num > 0.0 ? (double)INFINITY : 0.0);
  }
}

cudaError_t launch_output_error_final(const double* part, int nslots, double* err,
                                      cudaStream_t st) {
  return launch_pdl(output_error_final_kernel, dim3(1), dim3(kErrThreads), 0, st, part, nslots,
                    err);
}

cudaError_t launch_output_error(const float* y, const float* y_ref, int64_t n, double* scratch,
                                double* err, cudaStream_t st) {
  const int blocks = output_error_blocks(n);
  cudaError_t e = launch_pdl(output_error_kernel, dim3((unsigned)blocks), dim3(kErrThreads), 0,
                             st, y, y_ref, n, scratch);
  if (e != cudaSuccess) return e;
  return launch_output_error_final(scratch, blocks, err, st);
}

// ============================================================ producer fold
// 1/s folded into a producing linear: its per-output-channel scale and bias
// divided by s (one fp32 division each, [review] §5.5).
__global__ void fold_producer_kernel(const float* __restrict__ s, int64_t K, float* w_scale,
                                     float* bias) {
  pdl_launch_dependents();
  pdl_wait();
  for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < K;
       k += (int64_t)gridDim.x * blockDim.x) {
    const float sk = s[k];
    w_scale[k] = __fdiv_rn(w_scale[k], sk);
    if (bias) bias[k] = __fdiv_rn(bias[k], sk);
  }
}

cudaError_t launch_fold_producer(const float* s, int64_t K, float* w_scale, float* bias,
                                 cudaStream_t st) {
  int64_t blocks = (K + 255) / 256;
  if (blocks > 1024) blocks = 1024;
  return launch_pdl(fold_producer_kernel, dim3((unsigned)blocks), dim3(256), 0, st, s, K,
                    w_scale, bias);
}

// ============================================================ LayerNorm fold
// gamma' = gamma / s, beta' = beta / s ([embedded] §二), fp32 division.  The
// weight fold's row kernel does this itself; this kernel serves calls with
// no weight rows.
__global__ void fold_ln_kernel(const float* __restrict__ gamma, const float* __restrict__ beta,
                               const float* __restrict__ s, int64_t K,
                               float* __restrict__ gamma_out, float* __restrict__ beta_out) {
  pdl_launch_dependents();
  pdl_wait();
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
  return launch_pdl(fold_ln_kernel, dim3((unsigned)blocks), dim3(256), 0, st, gamma, beta, s, K,
                    gamma_out, beta_out);
}

}  // namespace sq
