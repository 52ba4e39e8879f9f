// probe.cu -- measurement support: the INT8 tensor-core issue rate of this
// GPU, the denominator of the large-M GEMM's roofline.
//
// One CTA per SM keeps a 128 x 256 INT32 accumulator in TMEM and issues
// tcgen05.mma kind::i8 steps of 128 x 256 x 32 back to back from operand
// tiles that sit in shared memory (filled once with pseudo-random bytes, so
// the multipliers switch as they would on real data).  Nothing else runs:
// no global-memory traffic, no epilogue.  The caller times the launch; the
// rate is 2 * 128 * 256 * 128 multiply-adds' worth of ops per k-block per
// CTA.  The one wait (for the last MMA) is bounded.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "sq_device.cuh"
#include "sq_internal.h"
#include "tc_ptx.cuh"

namespace sq {
namespace {

constexpr int kPA = 128 * 128;  // A tile: 128 rows x 128 bytes of K
constexpr int kPB = 256 * 128;  // B tile: 256 rows x 128 bytes of K
// more shared memory than two CTAs could share: one CTA per SM
constexpr size_t kProbeSmem = 120 * 1024;
constexpr uint64_t kProbeWaitNs = 4000000000ull;

__global__ void __launch_bounds__(128, 1) mma_i8_probe_kernel(int64_t kblocks, unsigned int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kPA + kPB);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
  const int warp = threadIdx.x >> 5;

  // operand bytes from a multiplicative hash of the word index
  uint32_t* w = reinterpret_cast<uint32_t*>(smem);
  for (int i = threadIdx.x; i < (kPA + kPB) / 4; i += blockDim.x)
    w[i] = (uint32_t)(i + 1 + blockIdx.x * 7919u) * 2654435761u;
  tc::fence_proxy_async_smem();  // generic writes before the MMA's reads
  if (threadIdx.x == 0) {
    tc::mbar_init(tc::smem_u32(bar), 1);
    tc::mbar_fence_init();
  }
  if (warp == 0) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), 256);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && tc::elect_one()) {
    constexpr uint32_t idesc = tc::idesc_i8(128, 256);
    const uint32_t a0 = tc::smem_u32(smem), b0 = tc::smem_u32(smem + kPA);
    for (int64_t kb = 0; kb < kblocks; ++kb) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        tc::mma_i8(tmem, tc::desc_k_sw128(a0 + k * 32), tc::desc_k_sw128(b0 + k * 32), idesc,
                   (kb | k) != 0);
    }
    tc::mma_commit(tc::smem_u32(bar));
    int never = 0;
    tc::mbar_wait(tc::smem_u32(bar), 0, &never, kProbeWaitNs, status);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 256);
  }
}

// The same over CTA pairs: clusters of two CTAs, the even CTA issuing
// 256 x 256 x 32 tcgen05.mma.cta_group::2.kind::i8 steps that read A from
// both CTAs' shared memory (128 rows each) and B from both (128 rows each),
// each CTA's TMEM holding its 128 accumulator rows.  Same work per SM per
// step as the single-CTA probe.
__global__ void __launch_bounds__(128, 1) mma_i8_pair_probe_kernel(int64_t kblocks,
                                                                   unsigned int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  constexpr int kA = 128 * 128, kB = 128 * 128;  // this CTA's halves
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kA + kB);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 1);
  const int warp = threadIdx.x >> 5;
  const bool leader = tc::cluster_ctarank() == 0;

  uint32_t* w = reinterpret_cast<uint32_t*>(smem);
  for (int i = threadIdx.x; i < (kA + kB) / 4; i += blockDim.x)
    w[i] = (uint32_t)(i + 1 + blockIdx.x * 7919u) * 2654435761u;
  tc::fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    tc::mbar_init(tc::smem_u32(bar), 1);
    tc::mbar_fence_init();
  }
  if (warp == 0) {
    tc::tmem_alloc_pair(tc::smem_u32(tmem_slot), 256);
    tc::tmem_relinquish_pair();
  }
  tc::tc_fence_before();
  tc::cluster_sync();  // both CTAs' operands and barriers are ready
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (leader && warp == 0 && tc::elect_one()) {
    constexpr uint32_t idesc = tc::idesc_i8(256, 256);
    const uint32_t a0 = tc::smem_u32(smem), b0 = tc::smem_u32(smem + kA);
    for (int64_t kb = 0; kb < kblocks; ++kb) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        tc::mma_i8_pair(tmem, tc::desc_k_sw128(a0 + k * 32), tc::desc_k_sw128(b0 + k * 32), idesc,
                        (kb | k) != 0);
    }
    tc::mma_commit_pair(tc::smem_u32(bar), 0x1);
    int never = 0;
    tc::mbar_wait(tc::smem_u32(bar), 0, &never, kProbeWaitNs, status);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::cluster_sync();  // the even CTA's MMAs, which read this CTA's operands, are done
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc_pair(tmem, 256);
  }
}

}  // namespace

cudaError_t launch_mma_pair_probe(int64_t kblocks, int pairs, cudaStream_t st) {
  unsigned int* sw = status_word();
  if (!sw) return cudaErrorInvalidDevice;
  static std::once_flag once[64];
  static cudaError_t attr_err[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) return e != cudaSuccess ? e : cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] {
    attr_err[dev] = cudaFuncSetAttribute(mma_i8_pair_probe_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kProbeSmem);
  });
  if (attr_err[dev] != cudaSuccess) return attr_err[dev];
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = kProbeSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mma_i8_pair_probe_kernel, kblocks, sw);
}

cudaError_t launch_mma_probe(int64_t kblocks, int grid, cudaStream_t st) {
  unsigned int* sw = status_word();
  if (!sw) return cudaErrorInvalidDevice;
  static std::once_flag once[64];
  static cudaError_t attr_err[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) return e != cudaSuccess ? e : cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] {
    attr_err[dev] = cudaFuncSetAttribute(mma_i8_probe_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kProbeSmem);
  });
  if (attr_err[dev] != cudaSuccess) return attr_err[dev];
  mma_i8_probe_kernel<<<grid, 128, kProbeSmem, st>>>(kblocks, sw);
  return cudaGetLastError();
}

}  // namespace sq
