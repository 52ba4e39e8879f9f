// gemm.cu -- INT8 x INT8 -> INT32 GEMM with the dequantizing epilogue of the
// smoothed W8A8 linear layer, on the sm_100a tensor cores (tcgen05.mma
// kind::i8, TMA-fed shared-memory tiles, INT32 accumulators in TMEM).
//
//   acc[t,n] = sum_k xq[t,k] * wq[n,k]                 (exact INT32)
//   y[t,n]   = (float)acc[t,n] * (as_t * w_scale[n])   (fp32, then bf16 RNE)
//
// Sources: "SmoothQuant：大型语言模型的精准高效训练后量化 — 深度技术评审" §2.6
// and Fig. 3 (an INT8 GEMM can take scales only on its outer dimensions: one
// per token row, one per output channel), §5.6 and Fig. 6 (linear layers run
// in INT8); "嵌入式 SLM 动态权重量化：SmoothQuant 激活异常值迁移与 INT8 部署实战"
// §三 (integer inner product, then one float rescale per output).
//
// Large-M kernel: persistent, one CTA per SM, 128 x 256 output tiles, 128-byte
// K steps, a 4-stage TMA ring, and two TMEM accumulators (2 x 256 columns) so
// the epilogue of one tile overlaps the main loop of the next.  Warp roles:
// warp 0 issues TMA loads, warp 1 issues the MMAs (one elected thread), warps
// 2-5 drain TMEM, dequantize and store.  Every mbarrier wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "sq_device.cuh"
#include "sq_internal.h"
#include "tc_ptx.cuh"

namespace sq {

namespace {

constexpr int BM = 128;     // token rows per tile (MMA M)
constexpr int BN = 256;     // output channels per tile (MMA N)
constexpr int BK = 128;     // bytes of K per stage = one 128B swizzle row
constexpr int UK = 32;      // K per tcgen05.mma kind::i8
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK;
constexpr int B_BYTES = BN * BK;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr int GROUP_M = 16;  // tile raster: 16 row blocks share each column sweep
constexpr uint64_t kWaitNs = 4000000000ull;   // 4 s: far above any pipeline step
constexpr uint64_t kDrainNs = 1000000000ull;  // waits for copies already in flight
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + 256;

struct Params {
  int M, N, K;
  int m_tiles, n_tiles, num_tiles, nk;
  const float* act_scale;
  int per_token;
  const float* w_scale;
  void* y;
  int32_t* acc;
  unsigned int* status;
};

__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int n_tiles, int& mb, int& nb) {
  const int per_group = GROUP_M * n_tiles;
  const int group = tile / per_group;
  const int first = group * GROUP_M;
  const int gm = min(m_tiles - first, GROUP_M);
  const int r = tile - group * per_group;
  mb = first + r % gm;
  nb = r / gm;
}

// Store 32 consecutive outputs of one row.  Fast path: 16-byte vector stores
// when the whole chunk is in range and rows stay 16-byte aligned.
template <bool BF16>
__device__ __forceinline__ void store_chunk(const Params& p, int row, int col0,
                                            const uint32_t (&r)[32], float as) {
  const bool full = col0 + 32 <= p.N;
  float ws[32];
  if (full) {
    const float4* w4 = reinterpret_cast<const float4*>(p.w_scale + col0);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 v = __ldg(w4 + i);
      ws[4 * i] = v.x; ws[4 * i + 1] = v.y; ws[4 * i + 2] = v.z; ws[4 * i + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) ws[i] = col0 + i < p.N ? __ldg(p.w_scale + col0 + i) : 0.0f;
  }
  float yv[32];
#pragma unroll
  for (int i = 0; i < 32; ++i)
    yv[i] = __fmul_rn(__int2float_rn((int)r[i]), __fmul_rn(as, ws[i]));
  const size_t base = (size_t)row * (size_t)p.N + (size_t)col0;
  if (BF16) {
    __nv_bfloat16* y = reinterpret_cast<__nv_bfloat16*>(p.y) + base;
    if (full && (p.N % 8) == 0) {
      uint32_t h[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        __nv_bfloat162 t = __floats2bfloat162_rn(yv[2 * i], yv[2 * i + 1]);
        h[i] = *reinterpret_cast<uint32_t*>(&t);
      }
      uint4* d = reinterpret_cast<uint4*>(y);
#pragma unroll
      for (int i = 0; i < 4; ++i) d[i] = make_uint4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (col0 + i < p.N) y[i] = __float2bfloat16_rn(yv[i]);
    }
  } else {
    float* y = reinterpret_cast<float*>(p.y) + base;
    if (full && (p.N % 4) == 0) {
      float4* d = reinterpret_cast<float4*>(y);
#pragma unroll
      for (int i = 0; i < 8; ++i) d[i] = make_float4(yv[4 * i], yv[4 * i + 1], yv[4 * i + 2], yv[4 * i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (col0 + i < p.N) y[i] = yv[i];
    }
  }
  if (p.acc) {
    int32_t* a = p.acc + base;
    if (full && (p.N % 4) == 0) {
      int4* d = reinterpret_cast<int4*>(a);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        d[i] = make_int4((int)r[4 * i], (int)r[4 * i + 1], (int)r[4 * i + 2], (int)r[4 * i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (col0 + i < p.N) a[i] = (int)r[i];
    }
  }
}

template <bool BF16>
__global__ void __launch_bounds__(THREADS, 1)
gemm_w8a8_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto full_bar = [&](int s) { return tc::smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return tc::smem_u32(bars + STAGES + s); };
  auto tfull_bar = [&](int b) { return tc::smem_u32(bars + 2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return tc::smem_u32(bars + 2 * STAGES + 2 + b); };
  const uint32_t drain_bar = tc::smem_u32(bars + 2 * STAGES + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(full_bar(s), 1);
      tc::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(tfull_bar(b), 1);
      tc::mbar_init(tempty_bar(b), 4);  // one arrival per epilogue warp
    }
    tc::mbar_init(drain_bar, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
    tc::tma_prefetch_desc(&tmA);
    tc::tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (tc::elect_one()) {
      uint32_t stage = 0, phase = 0, issued = 0, issued_par = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile, p.m_tiles, p.n_tiles, mb, nb);
        for (int kb = 0; kb < p.nk; ++kb) {
          if (!tc::mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, kWaitNs, p.status)) {
            ok = false;
            break;
          }
          tc::mbar_arrive_expect_tx(full_bar(stage), STAGE_BYTES);
          tc::tma_load_2d(tc::smem_u32(sA + stage * A_BYTES), &tmA, kb * BK, mb * BM, full_bar(stage));
          tc::tma_load_2d(tc::smem_u32(sB + stage * B_BYTES), &tmB, kb * BK, nb * BN, full_bar(stage));
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // let every load already issued land before the CTA exits
        int never = 0;
        for (int s = 0; s < STAGES; ++s)
          if (issued & (1u << s))
            tc::mbar_wait(full_bar(s), (issued_par >> s) & 1u, &never, kDrainNs, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (tc::elect_one()) {
      constexpr uint32_t idesc = tc::idesc_i8(BM, BN);
      uint32_t stage = 0, phase = 0, abuf = 0, aphase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        if (!tc::mbar_wait(tempty_bar(abuf), aphase ^ 1u, abort_flag, kWaitNs, p.status)) {
          ok = false;
          break;
        }
        tc::tc_fence_after();
        const uint32_t d = tmem_base + abuf * BN;
        for (int kb = 0; kb < p.nk; ++kb) {
          if (!tc::mbar_wait(full_bar(stage), phase, abort_flag, kWaitNs, p.status)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t a0 = tc::smem_u32(sA + stage * A_BYTES);
          const uint32_t b0 = tc::smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / UK; ++k)
            tc::mma_i8(d, tc::desc_k_sw128(a0 + k * UK), tc::desc_k_sw128(b0 + k * UK), idesc,
                       (kb | k) != 0);
          tc::mma_commit(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc::mma_commit(tfull_bar(abuf));
        abuf ^= 1u;
        if (abuf == 0) aphase ^= 1u;
      }
      // every MMA issued so far must finish before TMEM is released
      tc::mma_commit(drain_bar);
      int never = 0;
      tc::mbar_wait(drain_bar, 0, &never, kDrainNs, p.status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // this warp may read TMEM lanes 32*quarter..+31
    uint32_t abuf = 0, aphase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      int mb, nb;
      tile_coords(tile, p.m_tiles, p.n_tiles, mb, nb);
      if (!tc::mbar_wait(tfull_bar(abuf), aphase, abort_flag, kWaitNs, p.status)) break;
      tc::tc_fence_after();
      const int row = mb * BM + quarter * 32 + lane;
      const bool row_ok = row < p.M;
      const float as = p.per_token ? (row_ok ? __ldg(p.act_scale + row) : 0.0f) : __ldg(p.act_scale);
      const uint32_t taddr = tmem_base + abuf * BN + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tc::tmem_ld32(taddr + c * 32, r);
        tc::tmem_ld_wait();
        const int col0 = nb * BN + c * 32;
        if (row_ok && col0 < p.N) store_chunk<BF16>(p, row, col0, r, as);
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(tempty_bar(abuf));
      abuf ^= 1u;
      if (abuf == 0) aphase ^= 1u;
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// 2-D int8 tensor [rows, inner] (row stride = inner bytes), box
// [box_rows, 128 bytes], 128-byte swizzle, zero fill out of bounds.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool BF16>
cudaError_t launch_tc(const CUtensorMap& ta, const CUtensorMap& tb, const Params& p, int grid,
                      cudaStream_t st) {
  static std::once_flag once[64];
  static cudaError_t attr_err[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) return e != cudaSuccess ? e : cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] {
    attr_err[dev] = cudaFuncSetAttribute(gemm_w8a8_tc_kernel<BF16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
  });
  if (attr_err[dev] != cudaSuccess) return attr_err[dev];
  gemm_w8a8_tc_kernel<BF16><<<grid, THREADS, SMEM_BYTES, st>>>(ta, tb, p);
  return cudaGetLastError();
}

}  // namespace

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  (void)M; (void)N; (void)K;
  return 0;
}

sq_status launch_gemm(const GemmArgs& a, cudaStream_t st) {
  unsigned int* sw = status_word();
  if (!sw) return fail(SQ_ERR_CUDA, "sq_gemm_w8a8: device status word unavailable");
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, a.xq, (uint64_t)a.K, (uint64_t)a.M, BM) ||
      !make_tmap(&tb, a.wq, (uint64_t)a.K, (uint64_t)a.N, BN))
    return fail(SQ_ERR_CUDA, "sq_gemm_w8a8: cuTensorMapEncodeTiled failed");
  Params p{};
  p.M = (int)a.M; p.N = (int)a.N; p.K = (int)a.K;
  p.m_tiles = (int)((a.M + BM - 1) / BM);
  p.n_tiles = (int)((a.N + BN - 1) / BN);
  p.num_tiles = p.m_tiles * p.n_tiles;
  p.nk = (int)((a.K + BK - 1) / BK);
  p.act_scale = a.act_scale;
  p.per_token = a.act_per_token;
  p.w_scale = a.w_scale;
  p.y = a.y;
  p.acc = a.acc_out;
  p.status = sw;
  int grid = sm_count();
  if (grid > p.num_tiles) grid = p.num_tiles;
  cudaError_t e = a.yt == SQ_BF16 ? launch_tc<true>(ta, tb, p, grid, st)
                                  : launch_tc<false>(ta, tb, p, grid, st);
  if (e != cudaSuccess) return fail(SQ_ERR_CUDA, "sq_gemm_w8a8: %s", cudaGetErrorString(e));
  return SQ_OK;
}

}  // namespace sq
