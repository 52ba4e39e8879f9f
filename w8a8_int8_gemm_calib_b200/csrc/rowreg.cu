// rowreg.cu -- the static per-tensor activation quantizer without a
// LayerNorm in front (codes of x * (1/s) with one step for the whole call),
// with whole bf16 rows held in registers.
//
// Sources:
//   [review]   "SmoothQuant：大型语言模型的精准高效训练后量化 — 深度技术评审"
//              §2.2 (symmetric quantizer, round to nearest), §2.5-2.6
//              (static per-tensor step)
//   [embedded] "嵌入式 SLM 动态权重量化：SmoothQuant 激活异常值迁移与 INT8 部署实战"
//              §二 (per-tensor INT8 of the smoothed activations)
//
// Design.  A CTA of NT threads works on whole rows, dealt to the CTAs
// round-robin (row = CTA + i * grid).  Thread t owns the 8-element chunks
// t, t + NT, ... (CPT of them) of every row and reads them with 16-byte loads
// at L2.  A step covers U rows; the next step's loads are issued before the
// current step is quantized, so one step's bytes are always in flight.  The
// column multipliers sit in registers (CPT <= 2) or in shared memory.  Each
// element is independent (one step for the whole call): no barrier after
// the prologue.  Against the column-strip stream (rowops.cu) whole rows
// write their codes as long contiguous runs: 16384 x 8192 bf16 takes 76 us
// instead of 80.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "launch.cuh"
#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {

namespace {

constexpr int kMaxSmemMul = 20480;  // columns whose multipliers fit the shared-memory path

template <int NT, int CPT, int U, bool MREG>
__global__ void __launch_bounds__(NT, 1) rowreg_static_kernel(const RowArgs a) {
  extern __shared__ __align__(16) float msm[];
  pdl_launch_dependents();
  pdl_wait();
  const int tid = threadIdx.x;
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
    __syncthreads();
  }

  const float inv = __fdiv_rn(1.0f, __ldcg(a.scale));
  const bool count = a.n_clipped != nullptr;
  unsigned clipped = 0;
  for (int64_t r = r0; r < nT; r += U * RS) {
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int i = 0; i < CPT; ++i) cur[u][i] = pf[u][i];
    load_step(pf, row_of(r, U));
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t row = row_of(r, u);
#pragma unroll
      for (int i = 0; i < CPT; ++i) {
        const int c = tid + i * NT;
        if (c < nch && row < nT) {
          float v[8];
          unpack(cur[u][i], v);
          if (has_mul) {
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
          uint32_t b[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) b[e] = qbits(v[e], inv, count, clipped);
          if (in_bounds(row * K + (int64_t)c * 8, 8, size, a.status))
            store_codes(a.q + row * K + (int64_t)c * 8, b);
        }
      }
    }
  }
  if (count) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) clipped += __shfl_xor_sync(0xffffffffu, clipped, o);
    if ((tid & 31) == 0 && clipped) atomicAdd(a.n_clipped, (unsigned long long)clipped);
  }
}

template <int NT, int CPT, int U, bool MREG>
cudaError_t launch_t(const RowArgs& a, cudaStream_t st) {
  auto kern = rowreg_static_kernel<NT, CPT, U, MREG>;
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
  int64_t grid = sm_count();
  if (grid > a.T) grid = a.T;
  return launch_pdl(kern, dim3((unsigned)grid), dim3(NT), smem, st, a);
}

}  // namespace

bool rowreg_fits(int64_t K, sq_dtype xt, RowMode mode, bool ln) {
  return !ln && xt == SQ_BF16 && mode == ROW_STATIC && K % 8 == 0 && K / 8 <= 2560;
}

cudaError_t launch_rowreg(const RowArgs& a, RowMode mode, cudaStream_t st) {
  if (mode != ROW_STATIC) return cudaErrorInvalidValue;
  if (a.T <= 0) return cudaSuccess;
  const int64_t nch = a.K / 8;
  // up to 8192 columns: 512 threads, two rows a step, the multipliers in
  // registers; up to 20480: 640 threads of 4 chunks, one row a step, the
  // multipliers in shared memory
  if (nch <= 512) return launch_t<512, 1, 2, true>(a, st);
  if (nch <= 1024) return launch_t<512, 2, 2, true>(a, st);
  if (nch <= 2560) return launch_t<640, 4, 1, false>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace sq
