// rowreg.cu -- the row quantizers that have no LayerNorm in front, with each
// row held in registers: the weight fold (W * s quantized per output
// channel), the activation quantizer x * (1/s) with a step per token or one
// static step, and the peak pass of per-tensor dynamic quantization.
//
// Sources:
//   [review]   "SmoothQuant：大型语言模型的精准高效训练后量化 — 深度技术评审"
//              §2.2 (symmetric quantizer, step max|X|/127, round to nearest),
//              §2.5-2.6 (per-tensor static and per-token dynamic steps)
//   [embedded] "嵌入式 SLM 动态权重量化：SmoothQuant 激活异常值迁移与 INT8 部署实战"
//              §二 (W * diag(s) quantized with a static INT8 step per output channel)
//
// Design.  A CTA of NT threads works on whole bf16 rows, dealt to the CTAs
// round-robin (row = CTA + i * grid).  Thread t owns the 8-element chunks
// t, t + NT, ... (CPT of them) of every row it touches and reads them with
// 16-byte loads at L2.  A step covers U rows; the loads of the next step are
// issued before the current step is worked on, so one step's bytes are
// always in flight while the previous step is quantized.  The column
// multipliers sit in registers (CPT <= 2) or in shared memory.
//
// A step per row needs the row's peak first: each warp reduces its part
// (redux), the partials meet in shared memory behind one barrier per step,
// double-buffered so that the next step needs no second barrier.  The peak
// is taken with NaN propagated; a non-finite result (rare) falls back to the
// NaN-skipping peak with one more barrier, uniformly over the CTA.
//
// Measured against the shared-memory row ring (rowpipe.cu) on the same rows:
// 4096 x 20480 bf16 per token 57 us against 66, 16384 x 8192 static 76 against
// 80 (column strips), 28672 x 8192 per row 121 against 125.  Keeping a
// second step in flight (three register sets) or recomputing y instead of
// keeping it (for two CTAs per SM at 20480 columns) measured slower.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "launch.cuh"
#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {

namespace {

constexpr int kMaxSmemMul = 20480;  // columns whose multipliers fit the shared-memory path

template <int NT, int CPT, int U, int MODE, bool MREG, int NB>
__global__ void __launch_bounds__(NT, NB) rowreg_kernel(const RowArgs a) {
  constexpr int NW = NT / 32;
  constexpr int NWP = (NW + 3) / 4 * 4;  // partial rows padded to 16 bytes (pads = 0)
  extern __shared__ __align__(16) float msm[];
  __shared__ __align__(16) float red[2][U][NWP];
  __shared__ float red2[NW];
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (NWP != NW && tid < 2 * U * NWP) (&red[0][0][0])[tid] = 0.0f;

  const uint16_t* x = static_cast<const uint16_t*>(a.x);
  const int64_t K = a.K, nT = a.T, size = a.T * a.K;
  const int nch = (int)(K >> 3);
  const int64_t r0 = blockIdx.x, RS = gridDim.x;  // rows r0, r0 + RS, ...
  const bool has_mul = a.mul != nullptr;
  auto row_of = [&](int64_t r, int u) { return r + (int64_t)u * RS; };

  // the first step's rows go in flight before anything else is staged
  Raw8<uint16_t> pf[U][CPT], cur[U][CPT];
  auto load_step = [&](Raw8<uint16_t> (&b)[U][CPT], int64_t r) {
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int i = 0; i < CPT; ++i) {
        const int c = tid + i * NT;
        const int64_t row = row_of(r, u);
        b[u][i] = Raw8<uint16_t>{};
        if (c < nch && row < nT && in_bounds(row * K + (int64_t)c * 8, 8, size, a.status))
          load_raw(x + row * K + (int64_t)c * 8, b[u][i]);
      }
  };
  load_step(pf, r0);

  float mr[MREG ? CPT : 1][8];
  if constexpr (MREG) {
#pragma unroll
    for (int i = 0; i < CPT; ++i) {
      const int c = tid + i * NT;
#pragma unroll
      for (int e = 0; e < 8; ++e) mr[i][e] = 1.0f;
      if (c < nch && has_mul) load8(a.mul + (int64_t)c * 8, mr[i]);
    }
  } else {
    for (int64_t k = tid; k < K; k += NT) msm[k] = has_mul ? __ldcg(a.mul + k) : 1.0f;
  }
  fold_columns(a.mul, a.fold_g, a.fold_b, a.fold_g_out, a.fold_b_out, K, tid, NT);
  __syncthreads();

  // y = x * m for chunk i (column chunk c) of a raw row
  auto ychunk = [&](const Raw8<uint16_t>& raw, int i, int c, float (&v)[8]) {
    unpack(raw, v);
    if (has_mul && c < nch) {
      float m[8];
      if constexpr (MREG) {
#pragma unroll
        for (int e = 0; e < 8; ++e) m[e] = mr[i][e];
      } else {
        const float4 p = *reinterpret_cast<const float4*>(msm + c * 8);
        const float4 q = *reinterpret_cast<const float4*>(msm + c * 8 + 4);
        m[0] = p.x; m[1] = p.y; m[2] = p.z; m[3] = p.w;
        m[4] = q.x; m[5] = q.y; m[6] = q.z; m[7] = q.w;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = __fmul_rn(v[e], m[e]);
    }
  };

  const float sinv = MODE == ROW_STATIC ? __fdiv_rn(1.0f, __ldcg(a.scale)) : 0.0f;
  const bool count = a.n_clipped != nullptr;
  unsigned clipped = 0;
  float pk = 0.0f;  // ROW_PEAK: running peak of |y| (NaN skipped)
  int par = 0;

  for (int64_t r = r0; r < nT; r += U * RS) {
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int i = 0; i < CPT; ++i) cur[u][i] = pf[u][i];
    load_step(pf, row_of(r, U));

    if constexpr (MODE == ROW_STATIC || MODE == ROW_PEAK) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t row = row_of(r, u);
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
          const int c = tid + i * NT;
          if (c < nch && row < nT) {
            float v[8];
            ychunk(cur[u][i], i, c, v);
            if constexpr (MODE == ROW_PEAK) {
#pragma unroll
              for (int e = 0; e < 8; ++e) pk = fmaxf(pk, fabsf(v[e]));
            } else {
              uint32_t b[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) b[e] = qbits(v[e], sinv, count, clipped);
              if (in_bounds(row * K + (int64_t)c * 8, 8, size, a.status))
                store_codes(a.q + row * K + (int64_t)c * 8, b);
            }
          }
        }
      }
    } else {
      // per-row step: y kept in registers between the peak and the codes
      float y[U][CPT][8];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float m4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
          ychunk(cur[u][i], i, tid + i * NT, y[u][i]);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            m4[e] = max_nan3(m4[e], fabsf(y[u][i][2 * e]), fabsf(y[u][i][2 * e + 1]));
        }
        const float w = warp_maxabs_nan(max_nan(max_nan3(m4[0], m4[1], m4[2]), m4[3]));
        if (lane == 0) red[par][u][warp] = w;
      }
      __syncthreads();
      float mx[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float m = 0.0f;
#pragma unroll
        for (int t = 0; t < NWP; t += 4) {
          const float4 p = *reinterpret_cast<const float4*>(&red[par][u][t]);
          m = max_nan(m, max_nan(max_nan3(p.x, p.y, p.z), p.w));
        }
        mx[u] = m;  // >= 0, or NaN
      }
      par ^= 1;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t row = row_of(r, u);
        if (row >= nT) break;  // uniform over the CTA
        float m = mx[u];
        const bool clean = m < INFINITY;  // false for inf and NaN, uniformly
        if (!clean) {
          // the peak over the non-NaN values
          float m2 = 0.0f;
#pragma unroll
          for (int i = 0; i < CPT; ++i)
#pragma unroll
            for (int e = 0; e < 8; ++e) m2 = fmaxf(m2, fabsf(y[u][i][e]));
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) m2 = fmaxf(m2, __shfl_xor_sync(0xffffffffu, m2, o));
          __syncthreads();  // red2 is free (read before this barrier)
          if (lane == 0) red2[warp] = m2;
          __syncthreads();
          m2 = 0.0f;
#pragma unroll
          for (int t = 0; t < NW; ++t) m2 = fmaxf(m2, red2[t]);
          m = m2;
        }
        const float delta = __fdiv_rn(fmaxf(m, 1e-7f), 127.0f);
        const float inv = __fdiv_rn(1.0f, delta);
        if (tid == 0 && in_bounds(row, 1, nT, a.status)) a.scale[row] = delta;
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
          const int c = tid + i * NT;
          if (c < nch) {
            uint32_t b[8];
            if (clean) {
              // |y * inv| <= 127 * (1 + 2^-23) < 127.5: rounds without a clamp
#pragma unroll
              for (int e = 0; e < 8; ++e)
                b[e] = __float_as_uint(__fadd_rn(__fmul_rn(y[u][i][e], inv), kRoundMagic));
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e) b[e] = qbits(y[u][i][e], inv, count, clipped);
            }
            if (in_bounds(row * K + (int64_t)c * 8, 8, size, a.status))
              store_codes(a.q + row * K + (int64_t)c * 8, b);
          }
        }
      }
    }
  }
  if constexpr (MODE == ROW_PEAK) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) pk = fmaxf(pk, __shfl_xor_sync(0xffffffffu, pk, o));
    if (lane == 0) atomicMax(reinterpret_cast<unsigned int*>(a.peak), __float_as_uint(pk));
  } else if (count) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) clipped += __shfl_xor_sync(0xffffffffu, clipped, o);
    if (lane == 0 && clipped) atomicAdd(a.n_clipped, (unsigned long long)clipped);
  }
}

template <int NT, int CPT, int U, int MODE, bool MREG, int NB>
cudaError_t launch_t(const RowArgs& a, cudaStream_t st) {
  auto kern = rowreg_kernel<NT, CPT, U, MODE, MREG, NB>;
  const size_t smem = MREG ? 0 : (size_t)a.K * sizeof(float);
  if (!MREG) {
    // the dynamic shared-memory limit is raised once per instantiation and
    // device, to the largest the shapes routed here need
    static std::once_flag once[64];
    static cudaError_t attr_err[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64)
      return e != cudaSuccess ? e : cudaErrorInvalidDevice;
    std::call_once(once[dev], [&] {
      attr_err[dev] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)(kMaxSmemMul * sizeof(float)));
    });
    if (attr_err[dev] != cudaSuccess) return attr_err[dev];
  }
  int64_t grid = (int64_t)sm_count() * NB;
  if (grid > a.T) grid = a.T;
  return launch_pdl(kern, dim3((unsigned)grid), dim3(NT), smem, st, a);
}

template <int MODE>
cudaError_t dispatch(const RowArgs& a, cudaStream_t st) {
  const int64_t nch = a.K / 8;
  // up to 8192 columns: 512 threads, the multipliers in registers; a
  // per-row step runs two CTAs per SM, one row per step each
  if constexpr (MODE == ROW_DYNAMIC) {
    if (nch <= 512) return launch_t<512, 1, 1, MODE, true, 2>(a, st);
    if (nch <= 1024) return launch_t<512, 2, 1, MODE, true, 2>(a, st);
  } else {
    if (nch <= 512) return launch_t<512, 1, 2, MODE, true, 1>(a, st);
    if (nch <= 1024) return launch_t<512, 2, 2, MODE, true, 1>(a, st);
  }
  // up to 20480 columns: 640 threads of 4 chunks, the multipliers in shared memory
  if (nch <= 2560) return launch_t<640, 4, 1, MODE, false, 1>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace

bool rowreg_fits(int64_t K, sq_dtype xt, RowMode mode, bool ln) {
  return !ln && xt == SQ_BF16 && K % 8 == 0 && K / 8 <= 2560 &&
         (mode == ROW_DYNAMIC || mode == ROW_STATIC || mode == ROW_PEAK);
}

cudaError_t launch_rowreg(const RowArgs& a, RowMode mode, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  switch (mode) {
    case ROW_DYNAMIC: return dispatch<ROW_DYNAMIC>(a, st);
    case ROW_STATIC: return dispatch<ROW_STATIC>(a, st);
    case ROW_PEAK: return dispatch<ROW_PEAK>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sq
