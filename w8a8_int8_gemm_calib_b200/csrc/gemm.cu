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
// 2-5 drain TMEM, dequantize and store (warps 2-13 when K is short and the
// epilogue sets the pace).  Every mbarrier wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <string.h>

#include "launch.cuh"
#include "sq_device.cuh"
#include "sq_internal.h"
#include "tc_ptx.cuh"

namespace sq {

namespace {

constexpr int BM = 128;     // token rows per tile (MMA M)
constexpr int BK = 128;     // bytes of K per stage = one 128B swizzle row
constexpr int UK = 32;      // K per tcgen05.mma kind::i8
constexpr int A_BYTES = BM * BK;
constexpr int THREADS = 192;  // small-M kernel: TMA, MMA and 4 epilogue warps
constexpr int GROUP_M = 16;  // tile raster: 16 row blocks share each column sweep
constexpr uint64_t kWaitNs = 4000000000ull;   // 4 s: far above any pipeline step
constexpr uint64_t kDrainNs = 1000000000ull;  // waits for copies already in flight
constexpr uint64_t kPairGraceNs = 2000000ull;   // after a time-out: the peer's copies land
// Output staging for the TMA-store epilogue: per epilogue warp, buffers of
// 32 rows x 64 bytes (32 bf16 or 16 fp32 columns), 64-byte swizzled.
constexpr int EPI_BUF = 32 * 64;

// Large-M tile shapes: 128 x TBN outputs per tile, TBN in {256, 192, 128};
// the host picks the one that fills the last wave of SMs best.  EPI_NB
// output staging buffers per epilogue warp (EPI_NB - 1 TMA stores in flight
// per warp; deeper staging was measured not to speed up output-bound
// shapes).  EPI_W epilogue warps, 4 or 12: with 12, three warps share each
// 32-lane quarter of the accumulator and take every third 32-column chunk,
// for short K, where the epilogue and not the main loop sets the tile time
// and one warp per quarter leaves it latency-bound.
template <int TBN, int EPI_NB = 2, int EPI_W = 4, bool PAIR = false>
struct TcCfg {
  static_assert(EPI_W == 4 || EPI_W == 12, "one or three warps per accumulator quarter");
  static constexpr int THREADS = 64 + 32 * EPI_W;  // TMA warp, MMA warp, epilogue
  // a CTA pair's tile is 256 x TBN: each CTA holds 128 rows of A and TBN/2
  // rows of B per stage
  static constexpr int TILE_M = PAIR ? 2 * BM : BM;
  static constexpr int B_ROWS = PAIR ? TBN / 2 : TBN;
  static constexpr int B_BYTES = B_ROWS * BK;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int EPI_BYTES = EPI_W * EPI_NB * EPI_BUF;
  // as many stages as fit: with 4 epilogue warps of 2 staging buffers, 4 at
  // 256 columns, 5 at 192, 6 at 128
  static constexpr int STAGES = (224 * 1024 - 2048 - EPI_BYTES) / STAGE;
  static constexpr uint32_t TMEM_COLS = 2 * TBN <= 256 ? 256 : 512;  // power of two
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + EPI_BYTES + 256;
  static_assert(STAGES >= 2, "two main-loop stages at least");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

struct Params {
  int M, N, K;
  int m_tiles, n_tiles, num_tiles, nk;
  int tiles_per_batch;  // m_tiles * n_tiles (num_tiles = batch * tiles_per_batch)
  int group;            // tile raster: row tiles per band (each band sweeps every column)
  int w_per_tensor;     // batched: one weight step per batch (w_scale[b])
  int tma_store;  // outputs leave through shared memory and TMA stores
  int64_t y_elems;  // elements of y (and acc): batch * M * N
  const float* act_scale;
  int per_token;
  const float* w_scale;
  const float* bias;  // [N] added after the dequantization, or NULL
  void* y;
  int32_t* acc;
  unsigned int* status;
  // error mode: the reference output [M, N] fp32 and the per-warp fp64 sums
  // (2 per epilogue warp of every CTA); y is not written
  const float* err_ref;
  double* err_part;
};

__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int n_tiles, int& mb, int& nb,
                                            int group_m = GROUP_M) {
  const int per_group = group_m * n_tiles;
  const int group = tile / per_group;
  const int first = group * group_m;
  const int gm = min(m_tiles - first, group_m);
  const int r = tile - group * per_group;
  mb = first + r % gm;
  nb = r / gm;
}

// 32 per-column values (scales or bias) starting at col0; 0 past N.
__device__ __forceinline__ void load_cols32(const float* src, int col0, int N, float (&v)[32]) {
  if (col0 + 32 <= N && ((reinterpret_cast<uintptr_t>(src + col0) & 15) == 0)) {
    const float4* s4 = reinterpret_cast<const float4*>(src + col0);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 t = __ldcg(s4 + i);
      v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = col0 + i < N ? __ldcg(src + col0 + i) : 0.0f;
  }
}

// (float)acc * (as * ws); a bias is added after it as a separate fp32
// rounding (the intrinsics are never fused into a multiply-add)
__device__ __forceinline__ float dequant(uint32_t acc, float as, float ws) {
  return __fmul_rn(__int2float_rn((int)acc), __fmul_rn(as, ws));
}

// The weight steps (and bias) of the 32 columns col0..col0+31 of batch b:
// ws per output channel (batch b's row of w_scale) or, for a batch with one
// weight step, wt = w_scale[b].  They are loaded before the chunk's
// accumulators, so that their L2 latency overlaps the TMEM load (measured:
// 16384 x 28672 x 8192 2382 -> 2264 us, attention scores 94.2 -> 92.2 us).
template <bool BATCH>
__device__ __forceinline__ void load_scales(const Params& p, int b, int col0, float wt,
                                            float (&ws)[32], float (&bs)[32]) {
  if (BATCH && p.w_per_tensor) {
#pragma unroll
    for (int i = 0; i < 32; ++i) ws[i] = wt;
  } else {
    load_cols32(p.w_scale + (BATCH ? (size_t)b * (size_t)p.N : (size_t)0), col0, p.N, ws);
  }
  if (p.bias) load_cols32(p.bias, col0, p.N, bs);
}
// The 32 outputs of one row: (float)acc * (as * ws[n]) (+ bias[n])
__device__ __forceinline__ void dequant_loaded(const Params& p, const uint32_t (&r)[32], float as,
                                               const float (&ws)[32], const float (&bs)[32],
                                               float (&yv)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) yv[i] = dequant(r[i], as, ws[i]);
  if (p.bias) {
#pragma unroll
    for (int i = 0; i < 32; ++i) yv[i] = __fadd_rn(yv[i], bs[i]);
  }
}

// Store 32 consecutive outputs (and accumulators) of output row yrow.  Fast
// path: 16-byte vector stores when the whole chunk is in range and rows
// stay 16-byte aligned.
template <bool BF16>
__device__ __forceinline__ void store_chunk(const Params& p, size_t yrow, int col0,
                                            const uint32_t (&r)[32], const float (&yv)[32]) {
  const bool full = col0 + 32 <= p.N;
  const size_t base = yrow * (size_t)p.N + (size_t)col0;
  if (!in_bounds((int64_t)base, min(32, p.N - col0), p.y_elems, p.status)) return;
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

// PAIR: a cluster of two CTAs (an even and an odd one, on two SMs) shares
// each 256 x TBN tile through tcgen05 .cta_group::2 -- every CTA loads 128
// rows of A and TBN/2 rows of B per k-block into its own shared memory, the
// even CTA issues the MMAs for both, and each CTA drains its own 128 rows of
// the accumulator.  Per SM that moves (16 + TBN/16) KB per k-block from L2
// instead of (16 + TBN/8) KB, for the same multiply-adds.  Both CTAs walk
// the same tile sequence; the odd CTA's loads complete on the even CTA's
// stage barriers, the even CTA's commits arrive on both CTAs' barriers, and
// both CTAs' epilogue warps release the accumulator on the even CTA's
// barrier.  No load is multicast.
template <bool BF16, int TBN, bool BATCH, int EPI_NB, int EPI_W, bool ERR, bool PAIR = false>
__global__ void __launch_bounds__(TcCfg<TBN, EPI_NB, EPI_W, PAIR>::THREADS, 1)
gemm_w8a8_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmY, const Params p) {
  static_assert(!PAIR || (!BATCH && !ERR), "CTA pairs serve the plain GEMM");
  using C = TcCfg<TBN, EPI_NB, EPI_W, PAIR>;
  constexpr int TILE_M = C::TILE_M;
  constexpr int B_ROWS = C::B_ROWS;
  constexpr int STAGES = C::STAGES;
  constexpr int B_BYTES = C::B_BYTES;
  constexpr int STAGE_BYTES = C::STAGE;
  constexpr uint32_t TMEM_COLS = C::TMEM_COLS;
  constexpr int BN = TBN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint8_t* sEpi = smem + STAGES * STAGE_BYTES;  // 1024-aligned
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + C::EPI_BYTES);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto full_bar = [&](int s) { return tc::smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return tc::smem_u32(bars + STAGES + s); };
  auto tfull_bar = [&](int b) { return tc::smem_u32(bars + 2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return tc::smem_u32(bars + 2 * STAGES + 2 + b); };
  const uint32_t drain_bar = tc::smem_u32(bars + 2 * STAGES + 4);
  // the CTA's place in its pair (0, the even CTA, issues the MMAs), and the
  // persistent loop's unit: one tile per CTA, or per pair
  const uint32_t rank = PAIR ? tc::cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int unit0 = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      tc::mbar_init(full_bar(s), 1);
      tc::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(tfull_bar(b), 1);
      // one arrival per epilogue warp (of both CTAs of a pair)
      tc::mbar_init(tempty_bar(b), PAIR ? 2 * EPI_W : EPI_W);
    }
    tc::mbar_init(drain_bar, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
    tc::tma_prefetch_desc(&tmA);
    tc::tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tc::tmem_alloc_pair(tc::smem_u32(tmem_slot), TMEM_COLS);
      tc::tmem_relinquish_pair();
    } else {
      tc::tmem_alloc(tc::smem_u32(tmem_slot), TMEM_COLS);
      tc::tmem_relinquish();
    }
  }
  tc::tc_fence_before();
  if constexpr (PAIR) tc::cluster_sync();  // the peer's barriers are initialised
  else __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // the prologue above touches no global memory

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (tc::elect_one()) {
      uint32_t stage = 0, phase = 0, issued = 0, issued_par = 0;
      bool ok = true;
      for (int tile = unit0; ok && tile < p.num_tiles; tile += units) {
        int mb, nb;
        const int b = BATCH ? tile / p.tiles_per_batch : 0;
        tile_coords(tile - b * p.tiles_per_batch, p.m_tiles, p.n_tiles, mb, nb, p.group);
        for (int kb = 0; kb < p.nk; ++kb) {
          if (!tc::mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, kWaitNs, p.status)) {
            ok = false;
            break;
          }
          if constexpr (PAIR) {
            // both CTAs' bytes complete on the even CTA's barrier, which
            // alone expects them
            const uint32_t fb = tc::mapa_shared(full_bar(stage), 0);
            if (leader) tc::mbar_arrive_expect_tx(full_bar(stage), 2 * STAGE_BYTES);
            tc::tma_load_2d_pair(tc::smem_u32(sA + stage * A_BYTES), &tmA, kb * BK,
                                 mb * TILE_M + (int)rank * BM, fb);
            tc::tma_load_2d_pair(tc::smem_u32(sB + stage * B_BYTES), &tmB, kb * BK,
                                 nb * BN + (int)rank * B_ROWS, fb);
            issued |= 1u << stage;
            issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
            if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            continue;
          }
          tc::mbar_arrive_expect_tx(full_bar(stage), STAGE_BYTES);
          if constexpr (BATCH) {
            tc::tma_load_3d(tc::smem_u32(sA + stage * A_BYTES), &tmA, kb * BK, mb * BM, b,
                            full_bar(stage));
            tc::tma_load_3d(tc::smem_u32(sB + stage * B_BYTES), &tmB, kb * BK, nb * BN, b,
                            full_bar(stage));
          } else {
            tc::tma_load_2d(tc::smem_u32(sA + stage * A_BYTES), &tmA, kb * BK, mb * BM,
                            full_bar(stage));
            tc::tma_load_2d(tc::smem_u32(sB + stage * B_BYTES), &tmB, kb * BK, nb * BN,
                            full_bar(stage));
          }
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // let every load already issued land before the CTA exits
        int never = 0;
        if (leader)
          for (int s = 0; s < STAGES; ++s)
            if (issued & (1u << s))
              tc::mbar_wait(full_bar(s), (issued_par >> s) & 1u, &never, kDrainNs, p.status);
        if constexpr (PAIR) {
          // the odd CTA's copies complete on the even CTA's barriers, which
          // it cannot wait on: a fixed grace period lets them land
          const uint64_t t0 = global_ns();
          while (global_ns() - t0 < kPairGraceNs) {
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (leader && tc::elect_one()) {
      constexpr uint32_t idesc = tc::idesc_i8(TILE_M, BN);
      uint32_t stage = 0, phase = 0, abuf = 0, aphase = 0;
      bool ok = true;
      for (int tile = unit0; ok && tile < p.num_tiles; tile += units) {
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
          for (int k = 0; k < BK / UK; ++k) {
            if constexpr (PAIR)
              tc::mma_i8_pair(d, tc::desc_k_sw128(a0 + k * UK), tc::desc_k_sw128(b0 + k * UK),
                              idesc, (kb | k) != 0);
            else
              tc::mma_i8(d, tc::desc_k_sw128(a0 + k * UK), tc::desc_k_sw128(b0 + k * UK), idesc,
                         (kb | k) != 0);
          }
          if constexpr (PAIR) tc::mma_commit_pair(empty_bar(stage), 0x3);
          else tc::mma_commit(empty_bar(stage));
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if constexpr (PAIR) tc::mma_commit_pair(tfull_bar(abuf), 0x3);
        else tc::mma_commit(tfull_bar(abuf));
        abuf ^= 1u;
        if (abuf == 0) aphase ^= 1u;
      }
      // every MMA issued so far must finish before TMEM is released
      if constexpr (PAIR) tc::mma_commit_pair(drain_bar, 0x1);
      else tc::mma_commit(drain_bar);
      int never = 0;
      tc::mbar_wait(drain_bar, 0, &never, kDrainNs, p.status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // this warp may read TMEM lanes 32*quarter..+31
    const int chunk0 = (warp - 2) >> 2;  // first of this warp's 32-column chunks
    // outputs are written once and never read back here: evict them first
    // from L2 so the operand bands stay resident
    const uint64_t y_policy = PAIR ? tc::l2_policy_evict_first() : 0ull;
    uint8_t* ebuf = sEpi + (warp - 2) * EPI_NB * EPI_BUF;
    uint32_t nstore = 0;  // TMA stores issued by this warp (selects the buffer)
    double e_num = 0.0, e_den = 0.0;  // error mode: this lane's sums
    uint32_t abuf = 0, aphase = 0;
    for (int tile = unit0; tile < p.num_tiles; tile += units) {
      int mb, nb;
      const int b = BATCH ? tile / p.tiles_per_batch : 0;
      tile_coords(tile - b * p.tiles_per_batch, p.m_tiles, p.n_tiles, mb, nb, p.group);
      if (!tc::mbar_wait(tfull_bar(abuf), aphase, abort_flag, kWaitNs, p.status)) break;
      tc::tc_fence_after();
      const int row0 = mb * TILE_M + (int)rank * BM + quarter * 32;
      const int row = row0 + lane;
      const bool row_ok = row < p.M;
      const size_t yrow = (size_t)b * (size_t)p.M + (size_t)row;  // output row of [batch*M, N]
      const float as = p.per_token ? (row_ok ? __ldcg(p.act_scale + yrow) : 0.0f)
                                   : __ldcg(p.act_scale + b);
      const uint32_t taddr = tmem_base + abuf * BN + ((uint32_t)(quarter * 32) << 16);
      const float wt = (BATCH && p.w_per_tensor) ? __ldcg(p.w_scale + b) : 0.0f;
#pragma unroll 1
      for (int c = chunk0; c < BN / 32; c += EPI_W / 4) {
        const int col0 = nb * BN + c * 32;
        float ws[32], bs[32];
        load_scales<BATCH>(p, b, col0, wt, ws, bs);  // in flight during the TMEM load
        uint32_t r[32];
        tc::tmem_ld32(taddr + c * 32, r);
        tc::tmem_ld_wait();
        // dequantize this lane's 32 outputs (row `row`, columns col0..+31)
        float yv[32];
        dequant_loaded(p, r, as, ws, bs, yv);
        if constexpr (ERR) {
          // (y - y_ref)^2 and y_ref^2 in fp64, y the fp32 output the store
          // path would write; columns past N hold y = 0 and read ref = 0
          if (row_ok && in_bounds((int64_t)(yrow * p.N), p.N, p.y_elems, p.status)) {
            float rv[32];
            load_cols32(p.err_ref + yrow * (size_t)p.N, col0, p.N, rv);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const double rr = (double)rv[i];
              const double d = (double)yv[i] - rr;
              e_num += d * d;
              e_den += rr * rr;
            }
          }
          continue;
        }
        if (!p.tma_store) {
          if (row_ok && col0 < p.N) store_chunk<BF16>(p, yrow, col0, r, yv);
          continue;
        }
        uint32_t wv[BF16 ? 16 : 32];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float y0 = yv[i];
          const float y1 = yv[i + 1];
          if (BF16) {
            __nv_bfloat162 t = __floats2bfloat162_rn(y0, y1);
            wv[i / 2] = *reinterpret_cast<uint32_t*>(&t);
          } else {
            wv[i] = __float_as_uint(y0);
            wv[i + 1] = __float_as_uint(y1);
          }
        }
        if (p.acc && row_ok && col0 < p.N &&
            in_bounds((int64_t)(yrow * p.N + col0), min(32, p.N - col0), p.y_elems, p.status)) {
          int32_t* a = p.acc + yrow * p.N + col0;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (col0 + i < p.N) a[i] = (int)r[i];
        }
        // 64-byte rows: one box for bf16 (32 columns), two for fp32 (16 each)
        const bool any = row0 < p.M && col0 < p.N;  // warp-uniform
#pragma unroll
        for (int h = 0; h < (BF16 ? 1 : 2); ++h) {
          uint8_t* buf = ebuf + (nstore % EPI_NB) * EPI_BUF;
          // the store that last read `buf` (EPI_NB stores ago) is done
          if (lane == 0) tc::bulk_wait_read<EPI_NB - 1>();
          __syncwarp();
          // row `lane`, 16-byte chunk k at chunk k ^ ((lane >> 1) & 3): the
          // 64-byte swizzle the tensor map undoes (conflict-free writes)
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int pk = k ^ ((lane >> 1) & 3);
            *reinterpret_cast<uint4*>(buf + lane * 64 + pk * 16) =
                make_uint4(wv[h * 16 + 4 * k], wv[h * 16 + 4 * k + 1], wv[h * 16 + 4 * k + 2],
                           wv[h * 16 + 4 * k + 3]);
          }
          tc::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int cx = col0 + h * 16;
            if (any && cx < p.N) {
              if constexpr (BATCH) tc::tma_store_3d(&tmY, tc::smem_u32(buf), cx, row0, b);
              else if constexpr (PAIR) tc::tma_store_2d_hint(&tmY, tc::smem_u32(buf), cx, row0, y_policy);
              else tc::tma_store_2d(&tmY, tc::smem_u32(buf), cx, row0);
            }
            tc::bulk_commit();
          }
          ++nstore;
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (PAIR) tc::mbar_arrive_cluster(tc::mapa_shared(tempty_bar(abuf), 0));
        else tc::mbar_arrive(tempty_bar(abuf));
      }
      abuf ^= 1u;
      if (abuf == 0) aphase ^= 1u;
    }
    if constexpr (ERR) {
      // a fixed butterfly, then one slot per warp: deterministic sums
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        e_num += __shfl_xor_sync(0xffffffffu, e_num, o);
        e_den += __shfl_xor_sync(0xffffffffu, e_den, o);
      }
      if (lane == 0) {
        const size_t slot = (size_t)blockIdx.x * EPI_W + (size_t)(warp - 2);
        p.err_part[2 * slot] = e_num;
        p.err_part[2 * slot + 1] = e_den;
      }
    }
    if (lane == 0) tc::bulk_wait_all();  // staged outputs written before the CTA exits
    __syncwarp();
  }

  tc::tc_fence_before();
  __syncthreads();
  // neither CTA of a pair leaves while the other may still reach its
  // barriers or shared memory
  if constexpr (PAIR) tc::cluster_sync();
  if (warp == 1) {
    tc::tc_fence_after();
    if constexpr (PAIR) tc::tmem_dealloc_pair(tmem_base, TMEM_COLS);
    else tc::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ====================================================================== small M
// Decode-shaped problems (up to 128 tokens, as use_small picks them) stream
// the weights through this kernel: the operands are swapped so that a
// 128-row block of Wq fills the MMA's M dimension and the (padded) tokens
// form its N dimension (NPAD in {8, 16, 32, 64, 128}).
// The work -- (weight tile, 128-byte k-block) units -- is split evenly over
// a persistent grid (stream-K): CTA g owns units [g*U/G, (g+1)*U/G).  A tile
// covered by one CTA is finished in place; otherwise every contributing CTA
// stores its INT32 partial tile into its own scratch slot, and the last one
// to arrive (an atomic counter per tile) sums the slots -- exact integer
// addition in any order -- and runs the epilogue.  No CTA ever waits for
// another one.
constexpr int SM_BM = 128;
constexpr int SM_A_BYTES = SM_BM * BK;

template <int NPAD>
struct SmallCfg {
  static constexpr int B_BYTES = NPAD * BK;
  static constexpr int STAGE = SM_A_BYTES + B_BYTES;
  static constexpr int STAGES = (200 * 1024) / STAGE > 12 ? 12 : (200 * 1024) / STAGE;
  static constexpr uint32_t TMEM_COLS = 2 * NPAD < 32 ? 32 : 2 * NPAD;
  static constexpr int CH = NPAD < 32 ? NPAD : 32;  // accumulator columns per TMEM load
  static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE + 512;
};

struct SmallParams {
  int M, N, K;
  int n_tiles, nk;
  int64_t units;  // n_tiles * nk
  int grid;
  const float* act_scale;
  int per_token;
  const float* w_scale;
  const float* bias;  // [N] added after the dequantization, or NULL
  void* y;
  int32_t* acc;
  int32_t* slots;           // [grid][2][M][128]
  unsigned int* counters;   // [n_tiles], zeroed before the launch
  unsigned int* status;
};

__device__ __forceinline__ int64_t unit_begin(int64_t g, const SmallParams& p) {
  return g * p.units / p.grid;
}
// the CTA whose range holds unit u
__device__ __forceinline__ int64_t unit_owner(int64_t u, const SmallParams& p) {
  return ((u + 1) * p.grid - 1) / p.units;
}

template <int CH>
__device__ __forceinline__ void tmem_ld_n(uint32_t taddr, uint32_t (&r)[CH]) {
  if constexpr (CH == 8) tc::tmem_ld8(taddr, r);
  else if constexpr (CH == 16) tc::tmem_ld16(taddr, r);
  else tc::tmem_ld32(taddr, r);
}

// y[t, n] (and acc[t, n]) for tokens t0 .. t0+CH-1 of output channel n
template <bool BF16, int CH>
__device__ __forceinline__ void small_store(const SmallParams& p, int n, int t0, const int32_t (&v)[CH]) {
  if (n >= p.N) return;
  const float ws = __ldcg(p.w_scale + n);
  const float bn = p.bias ? __ldcg(p.bias + n) : 0.0f;
#pragma unroll
  for (int i = 0; i < CH; ++i) {
    const int t = t0 + i;
    if (t < p.M) {
      const float as = __ldcg(p.act_scale + (p.per_token ? t : 0));
      float y = dequant((uint32_t)v[i], as, ws);
      if (p.bias) y = __fadd_rn(y, bn);
      const size_t o = (size_t)t * (size_t)p.N + (size_t)n;
      if (!in_bounds((int64_t)o, 1, (int64_t)p.M * p.N, p.status)) continue;
      if (BF16) reinterpret_cast<__nv_bfloat16*>(p.y)[o] = __float2bfloat16_rn(y);
      else reinterpret_cast<float*>(p.y)[o] = y;
      if (p.acc) p.acc[o] = v[i];
    }
  }
}

__device__ __forceinline__ void epi_bar() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}
// AND of v over the 128 epilogue threads of the small-M kernel (also a
// barrier among them), so that its four epilogue warps take the same branch
__device__ __forceinline__ bool epi_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, o;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred o, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, o;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

template <int NPAD, bool BF16>
__global__ void __launch_bounds__(THREADS, 1)
gemm_w8a8_smallm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                        const SmallParams p) {
  using C = SmallCfg<NPAD>;
  constexpr int S = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * SM_A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S * C::STAGE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto full_bar = [&](int s) { return tc::smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return tc::smem_u32(bars + S + s); };
  auto tfull_bar = [&](int b) { return tc::smem_u32(bars + 2 * S + b); };
  auto tempty_bar = [&](int b) { return tc::smem_u32(bars + 2 * S + 2 + b); };
  const uint32_t drain_bar = tc::smem_u32(bars + 2 * S + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(full_bar(s), 1);
      tc::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(tfull_bar(b), 1);
      tc::mbar_init(tempty_bar(b), 4);
    }
    tc::mbar_init(drain_bar, 1);
    *abort_flag = 0;
    tc::mbar_fence_init();
    tc::tma_prefetch_desc(&tmW);
    tc::tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_u32(tmem_slot), C::TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // the prologue above touches no global memory
  const int64_t ub = unit_begin(blockIdx.x, p), ue = unit_begin(blockIdx.x + 1, p);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (tc::elect_one()) {
      uint32_t stage = 0, phase = 0, issued = 0, issued_par = 0;
      bool ok = true;
      for (int64_t u = ub; ok && u < ue;) {
        const int tile = (int)(u / p.nk);
        const int kb0 = (int)(u % p.nk);
        const int kb1 = (int)min((int64_t)p.nk, kb0 + (ue - u));
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!tc::mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, kWaitNs, p.status)) {
            ok = false;
            break;
          }
          tc::mbar_arrive_expect_tx(full_bar(stage), C::STAGE);
          tc::tma_load_2d(tc::smem_u32(sA + stage * SM_A_BYTES), &tmW, kb * BK, tile * SM_BM,
                          full_bar(stage));
          tc::tma_load_2d(tc::smem_u32(sB + stage * C::B_BYTES), &tmX, kb * BK, 0, full_bar(stage));
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        u += kb1 - kb0;
      }
      if (!ok) {
        int never = 0;
        for (int s = 0; s < S; ++s)
          if (issued & (1u << s))
            tc::mbar_wait(full_bar(s), (issued_par >> s) & 1u, &never, kDrainNs, p.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (tc::elect_one()) {
      constexpr uint32_t idesc = tc::idesc_i8(SM_BM, NPAD);
      uint32_t stage = 0, phase = 0, abuf = 0, aphase = 0;
      bool ok = true;
      for (int64_t u = ub; ok && u < ue;) {
        const int kb0 = (int)(u % p.nk);
        const int kb1 = (int)min((int64_t)p.nk, kb0 + (ue - u));
        if (!tc::mbar_wait(tempty_bar(abuf), aphase ^ 1u, abort_flag, kWaitNs, p.status)) break;
        tc::tc_fence_after();
        const uint32_t d = tmem_base + abuf * NPAD;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!tc::mbar_wait(full_bar(stage), phase, abort_flag, kWaitNs, p.status)) {
            ok = false;
            break;
          }
          tc::tc_fence_after();
          const uint32_t a0 = tc::smem_u32(sA + stage * SM_A_BYTES);
          const uint32_t b0 = tc::smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / UK; ++k)
            tc::mma_i8(d, tc::desc_k_sw128(a0 + k * UK), tc::desc_k_sw128(b0 + k * UK), idesc,
                       (kb != kb0) || (k != 0));
          tc::mma_commit(empty_bar(stage));
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc::mma_commit(tfull_bar(abuf));
        abuf ^= 1u;
        if (abuf == 0) aphase ^= 1u;
        u += kb1 - kb0;
      }
      tc::mma_commit(drain_bar);
      int never = 0;
      tc::mbar_wait(drain_bar, 0, &never, kDrainNs, p.status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int rloc = quarter * 32 + lane;  // output channel within the tile
    const int64_t slot_elems = (int64_t)p.grid * 2 * p.M * SM_BM;  // the partial-tile slots
    uint32_t abuf = 0, aphase = 0;
    for (int64_t u = ub; u < ue;) {
      const int tile = (int)(u / p.nk);
      const int kb0 = (int)(u % p.nk);
      const int kb1 = (int)min((int64_t)p.nk, kb0 + (ue - u));
      const bool full = kb0 == 0 && kb1 == p.nk;
      const int which = u == ub ? 0 : 1;
      const bool got = tc::mbar_wait(tfull_bar(abuf), aphase, abort_flag, kWaitNs, p.status);
      if (!epi_and(got)) break;
      tc::tc_fence_after();
      const int n = tile * SM_BM + rloc;
      const uint32_t taddr = tmem_base + abuf * NPAD + ((uint32_t)(quarter * 32) << 16);
      int32_t* slot = p.slots + ((int64_t)blockIdx.x * 2 + which) * (int64_t)p.M * SM_BM;
#pragma unroll 1
      for (int c0 = 0; c0 < NPAD; c0 += C::CH) {
        uint32_t r[C::CH];
        tmem_ld_n<C::CH>(taddr + c0, r);
        tc::tmem_ld_wait();
        if (full) {
          int32_t v[C::CH];
#pragma unroll
          for (int i = 0; i < C::CH; ++i) v[i] = (int32_t)r[i];
          small_store<BF16, C::CH>(p, n, c0, v);
        } else {
#pragma unroll
          for (int i = 0; i < C::CH; ++i)
            if (c0 + i < p.M &&
                in_bounds((slot - p.slots) + (int64_t)(c0 + i) * SM_BM + rloc, 1, slot_elems, p.status))
              slot[(int64_t)(c0 + i) * SM_BM + rloc] = (int32_t)r[i];
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(tempty_bar(abuf));
      abuf ^= 1u;
      if (abuf == 0) aphase ^= 1u;
      if (!full) {
        // publish the partial tile, then count arrivals; the last one sums
        const int64_t gf = unit_owner((int64_t)tile * p.nk, p);
        const int64_t gl = unit_owner((int64_t)tile * p.nk + p.nk - 1, p);
        __threadfence();
        epi_bar();
        if (threadIdx.x == 64) {
          const unsigned prev = in_bounds(tile, 1, p.n_tiles, p.status)
                                    ? atomicAdd(p.counters + tile, 1u)
                                    : 0u;
          *last_flag = prev == (unsigned)(gl - gf);
        }
        epi_bar();
        const bool last = *last_flag != 0;
        epi_bar();  // every thread has read the flag before it is reused
        if (last) {
          __threadfence();
#pragma unroll 1
          for (int c0 = 0; c0 < p.M; c0 += C::CH) {
            int32_t v[C::CH];
#pragma unroll
            for (int i = 0; i < C::CH; ++i) v[i] = 0;
            for (int64_t g = gf; g <= gl; ++g) {
              const int wg = ((int)(unit_begin(g, p) / p.nk) == tile) ? 0 : 1;
              const int32_t* sl = p.slots + (g * 2 + wg) * (int64_t)p.M * SM_BM;
#pragma unroll
              for (int i = 0; i < C::CH; ++i)
                if (c0 + i < p.M &&
                    in_bounds((sl - p.slots) + (int64_t)(c0 + i) * SM_BM + rloc, 1, slot_elems, p.status))
                  v[i] += __ldcg(sl + (int64_t)(c0 + i) * SM_BM + rloc);
            }
            small_store<BF16, C::CH>(p, n, c0, v);
          }
        }
      }
      u += kb1 - kb0;
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem_base, C::TMEM_COLS);
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

// Output tensor map for the TMA-store epilogue: [rows, cols] of bf16/fp32,
// box 64 bytes x 32 rows, 64-byte swizzle.
bool make_tmap_out(CUtensorMap* m, void* base, uint64_t cols, uint64_t rows, bool bf16) {
  auto enc = encode_fn();
  if (!enc) return false;
  const uint64_t esz = bf16 ? 2 : 4;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * esz};
  cuuint32_t box[2] = {(cuuint32_t)(64 / esz), 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                   base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Batched operands: [batch, rows, inner] int8 (K-major rows), box
// [1, box_rows, 128 bytes], 128-byte swizzle, zero fill past each batch's
// rows and inner extent.
bool make_tmap3(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t batch,
                uint32_t box_rows) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {inner, rows, batch};
  cuuint64_t strides[2] = {inner, inner * rows};
  cuuint32_t box[3] = {(cuuint32_t)BK, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
// Batched output [batch, rows, cols]: stores clipped at each batch's edges.
bool make_tmap_out3(CUtensorMap* m, void* base, uint64_t cols, uint64_t rows, uint64_t batch,
                    bool bf16) {
  auto enc = encode_fn();
  if (!enc) return false;
  const uint64_t esz = bf16 ? 2 : 4;
  cuuint64_t dims[3] = {cols, rows, batch};
  cuuint64_t strides[2] = {cols * esz, cols * rows * esz};
  cuuint32_t box[3] = {(cuuint32_t)(64 / esz), 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
                   base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <bool BF16, int TBN, bool BATCH = false, int EPI_NB = 2, int EPI_W = 4, bool ERR = false>
cudaError_t launch_tc(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& ty,
                      const Params& p, int grid, cudaStream_t st) {
  using C = TcCfg<TBN, EPI_NB, EPI_W>;
  static std::once_flag once[64];
  static cudaError_t attr_err[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) return e != cudaSuccess ? e : cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] {
    attr_err[dev] = cudaFuncSetAttribute(gemm_w8a8_tc_kernel<BF16, TBN, BATCH, EPI_NB, EPI_W, ERR>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::SMEM);
  });
  if (attr_err[dev] != cudaSuccess) return attr_err[dev];
  return launch_pdl(gemm_w8a8_tc_kernel<BF16, TBN, BATCH, EPI_NB, EPI_W, ERR>, dim3(grid),
                    dim3(C::THREADS), C::SMEM, st, ta, tb, ty, p);
}

// The CTA-pair kernel: `pairs` clusters of two CTAs.  The number of pairs
// that can be resident at once is queried once per device and tile width;
// a persistent launch never asks for more.
template <bool BF16, int TBN>
cudaError_t launch_tc_pair(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& ty,
                           const Params& p, int pairs, cudaStream_t st) {
  using C = TcCfg<TBN, 2, 4, true>;
  auto kern = gemm_w8a8_tc_kernel<BF16, TBN, false, 2, 4, false, true>;
  static std::once_flag once[64];
  static cudaError_t attr_err[64];
  static int max_pairs[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) return e != cudaSuccess ? e : cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] {
    attr_err[dev] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::SMEM);
    if (attr_err[dev] != cudaSuccess) return;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * (unsigned)(sm_count() / 2));
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = C::SMEM;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    attr_err[dev] = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    max_pairs[dev] = n;
  });
  if (attr_err[dev] != cudaSuccess) return attr_err[dev];
  if (max_pairs[dev] < 1) return cudaErrorInvalidConfiguration;
  if (pairs > max_pairs[dev]) pairs = max_pairs[dev];
  return launch_pdl_cluster(kern, dim3(2 * pairs), dim3(C::THREADS), C::SMEM, st, 2u, ta, tb, ty,
                            p);
}

// Tile width for the large-M kernel: the per-tile time grows with the width,
// and a partly filled last wave costs a whole tile time, so take the width
// with the smaller (waves x width) -- plus a fixed per-tile cost.
int pick_tile_n(int64_t M, int64_t N, int sms, int64_t batch = 1, bool narrow = false) {
  const int64_t mt = (M + BM - 1) / BM;
  int best = 256;
  int64_t best_cost = -1;
  for (int tbn : {256, 192, 128}) {
    if (tbn == 128 && !narrow) continue;
    const int64_t tiles = batch * mt * ((N + tbn - 1) / tbn);
    const int64_t waves = (tiles + sms - 1) / sms;
    const int64_t cost = waves * (tbn + 16);
    if (best_cost < 0 || cost < best_cost) { best = tbn; best_cost = cost; }
  }
  return best;
}


// The large-M kernel for a tile width, output type and epilogue width (the
// 128-column tiles are only picked for batched calls).  Short K (at most
// four k-blocks) takes 12 epilogue warps: there a tile's main loop is a few
// MMAs and the epilogue sets the pace.
template <bool BATCH>
cudaError_t launch_tiles(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& ty,
                         const Params& p, int grid, int tbn, bool bf16, cudaStream_t st) {
  if (p.nk <= 4) {
    if (tbn == 256) return bf16 ? launch_tc<true, 256, BATCH, 2, 12>(ta, tb, ty, p, grid, st)
                                : launch_tc<false, 256, BATCH, 2, 12>(ta, tb, ty, p, grid, st);
    if (tbn == 192) return bf16 ? launch_tc<true, 192, BATCH, 2, 12>(ta, tb, ty, p, grid, st)
                                : launch_tc<false, 192, BATCH, 2, 12>(ta, tb, ty, p, grid, st);
    if constexpr (BATCH)
      return bf16 ? launch_tc<true, 128, BATCH, 2, 12>(ta, tb, ty, p, grid, st)
                  : launch_tc<false, 128, BATCH, 2, 12>(ta, tb, ty, p, grid, st);
  } else {
    if (tbn == 256) return bf16 ? launch_tc<true, 256, BATCH>(ta, tb, ty, p, grid, st)
                                : launch_tc<false, 256, BATCH>(ta, tb, ty, p, grid, st);
    if (tbn == 192) return bf16 ? launch_tc<true, 192, BATCH>(ta, tb, ty, p, grid, st)
                                : launch_tc<false, 192, BATCH>(ta, tb, ty, p, grid, st);
    if constexpr (BATCH)
      return bf16 ? launch_tc<true, 128, BATCH>(ta, tb, ty, p, grid, st)
                  : launch_tc<false, 128, BATCH>(ta, tb, ty, p, grid, st);
  }
  return cudaErrorInvalidValue;
}

// Tile width for the CTA-pair kernel (256-row tiles, one per pair of SMs),
// by the same wave cost as pick_tile_n.
int pick_tile_n_pair(int64_t M, int64_t N, int sms) {
  const int64_t mt = (M + 2 * BM - 1) / (2 * BM);
  const int64_t units = sms / 2;
  int best = 256;
  int64_t best_cost = -1;
  for (int tbn : {256, 192}) {
    const int64_t tiles = mt * ((N + tbn - 1) / tbn);
    const int64_t waves = (tiles + units - 1) / units;
    const int64_t cost = waves * (tbn + 16);
    if (best_cost < 0 || cost < best_cost) { best = tbn; best_cost = cost; }
  }
  return best;
}

// Row tiles per raster band of the CTA-pair kernel: the band's activation
// rows (tiles x 256 x K bytes) stay resident in L2 while the band sweeps
// every weight column, so the weights are read from DRAM once per band.
// About 32 MB of activations per band, 4 to 16 tiles (1024 to 4096 rows):
// measured on 16384 x 28672 x 8192, 4096-row bands take 2337 us against
// 2436-2457 us for 2048 and 2585 us for 8192.
int pair_band_tiles(int64_t K) {
  int64_t t = ((int64_t)32 << 20) / (2 * BM * (K > 0 ? K : 1));
  if (t > 16) t = 16;
  if (t < 4) t = 4;
  return (int)t;
}

// The plain GEMM takes CTA pairs for every M the large-M kernel serves,
// except short K (at most four k-blocks), where the epilogue and not the
// operand traffic sets the pace and the single-CTA kernel's twelve
// epilogue warps serve it better.
bool use_pair(int64_t M, int64_t K) { return M > 128 && (K + BK - 1) / BK > 4; }

constexpr int64_t kSmallMaxM = 128;

// Decode-shaped calls (M <= 128) stream the weights either way; the question
// is which kernel keeps every SM streaming.  Up to 8 tokens the stream-K
// kernel is always the faster one.  Beyond that, the persistent large-M
// kernel (one 128-row block, tiles across N) wins once its tiles fill every
// SM at least once: it fetches each activation k-block once per 192 or 256
// weight rows instead of once per 128, and keeps a deeper ring.  Measured on
// the 175B fc1 (49152 x 12288): 16 to 128 tokens in 104-107 us against
// 114-164 us.  Narrower outputs, whose large-M tiles would leave SMs idle,
// keep stream-K.
bool use_small(int64_t M, int64_t N) {
  if (M > kSmallMaxM) return false;
  if (M <= 8) return true;
  const int sms = sm_count();
  const int tbn = pick_tile_n(M, N, sms);
  return (N + tbn - 1) / tbn < sms;  // one row block: the tiles across N
}

int64_t small_grid(int64_t N, int64_t K) {
  const int64_t units = ((N + SM_BM - 1) / SM_BM) * ((K + BK - 1) / BK);
  const int64_t g = sm_count();
  return units < g ? units : g;
}

// Workspace of the small-M kernel: the per-tile arrival counters first
// (zeroed by every call), then the partial-tile slots [grid][2][M][128].
size_t counters_bytes(int64_t N) {
  const int64_t n_tiles = (N + SM_BM - 1) / SM_BM;
  return ((size_t)n_tiles * sizeof(unsigned int) + 255) & ~(size_t)255;
}

size_t gemm_workspace_bytes_impl(int64_t M, int64_t N, int64_t K) {
  if (!use_small(M, N)) return 0;
  const int64_t G = small_grid(N, K);
  return counters_bytes(N) + (size_t)G * 2 * (size_t)M * SM_BM * sizeof(int32_t);
}

template <int NPAD, bool BF16>
cudaError_t launch_small_t(const CUtensorMap& tw, const CUtensorMap& tx, const SmallParams& p,
                           cudaStream_t st) {
  static std::once_flag once[64];
  static cudaError_t attr_err[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) return e != cudaSuccess ? e : cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] {
    attr_err[dev] = cudaFuncSetAttribute(gemm_w8a8_smallm_kernel<NPAD, BF16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SmallCfg<NPAD>::SMEM);
  });
  if (attr_err[dev] != cudaSuccess) return attr_err[dev];
  return launch_pdl(gemm_w8a8_smallm_kernel<NPAD, BF16>, dim3(p.grid), dim3(THREADS),
                    SmallCfg<NPAD>::SMEM, st, tw, tx, p);
}

template <bool BF16>
cudaError_t launch_small(const GemmArgs& a, const SmallParams& p, cudaStream_t st) {
  const int npad = a.M <= 8 ? 8 : a.M <= 16 ? 16 : a.M <= 32 ? 32 : a.M <= 64 ? 64 : 128;
  CUtensorMap tw, tx;
  if (!make_tmap(&tw, a.wq, (uint64_t)a.K, (uint64_t)a.N, SM_BM) ||
      !make_tmap(&tx, a.xq, (uint64_t)a.K, (uint64_t)a.M, (uint32_t)npad))
    return cudaErrorInvalidValue;
  switch (npad) {
    case 8: return launch_small_t<8, BF16>(tw, tx, p, st);
    case 16: return launch_small_t<16, BF16>(tw, tx, p, st);
    case 32: return launch_small_t<32, BF16>(tw, tx, p, st);
    case 64: return launch_small_t<64, BF16>(tw, tx, p, st);
    default: return launch_small_t<128, BF16>(tw, tx, p, st);
  }
}

}  // namespace

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  return gemm_workspace_bytes_impl(M, N, K);
}

// Scratch of sq_gemm_w8a8_noalloc: a fixed array in device memory, reserved
// on every device that loads this library and kept until the process exits.
// All calls share it.  Host code only sees a stand-in for it, so its device
// address is looked up (cudaGetSymbolAddress) once per device, with that
// device current, the first time the entry point runs there.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};
}  // namespace

sq_status launch_gemm_noalloc(GemmArgs a, cudaStream_t st) {
  const size_t need = gemm_workspace_bytes_impl(a.M, a.N, a.K);
  if (need > kNoallocScratchBytes)
    return fail(SQ_ERR_WORKSPACE,
                "sq_gemm_w8a8_noalloc: M=%lld N=%lld K=%lld needs %zu bytes of scratch; the "
                "static scratch holds %zu (use sq_gemm_w8a8 with a workspace)",
                (long long)a.M, (long long)a.N, (long long)a.K, need, kNoallocScratchBytes);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(SQ_ERR_CUDA, "sq_gemm_w8a8_noalloc: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return fail(SQ_ERR_UNSUPPORTED, "sq_gemm_w8a8_noalloc: device %d", dev);
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
      void* ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
      if (e != cudaSuccess || !ptr)
        return fail(SQ_ERR_CUDA, "sq_gemm_w8a8_noalloc: cudaGetSymbolAddress: %s",
                    cudaGetErrorString(e));
      g_noalloc_ptr[dev] = ptr;
    }
    scratch = g_noalloc_ptr[dev];
  }
  a.workspace = need ? scratch : nullptr;
  a.workspace_bytes = need ? kNoallocScratchBytes : 0;
  return launch_gemm(a, st);
}

namespace {
// Tensor maps, parameters and grid of the large-M kernel for a plain GEMM
// (the output map and the store choice are the caller's).
struct LargeSetup {
  CUtensorMap ta, tb, ty;
  Params p;
  int tbn, grid;
  bool pair;  // grid counts CTA pairs
};
bool setup_large(const GemmArgs& a, unsigned int* sw, LargeSetup* L, bool allow_pair) {
  L->pair = allow_pair && use_pair(a.M, a.K);
  L->tbn = L->pair ? pick_tile_n_pair(a.M, a.N, sm_count()) : pick_tile_n(a.M, a.N, sm_count());
  const int tile_m = L->pair ? 2 * BM : BM;
  const int b_rows = L->pair ? L->tbn / 2 : L->tbn;
  if (!make_tmap(&L->ta, a.xq, (uint64_t)a.K, (uint64_t)a.M, BM) ||
      !make_tmap(&L->tb, a.wq, (uint64_t)a.K, (uint64_t)a.N, (uint32_t)b_rows))
    return false;
  memset(&L->ty, 0, sizeof L->ty);
  Params& p = L->p;
  p = Params{};
  p.M = (int)a.M; p.N = (int)a.N; p.K = (int)a.K;
  p.m_tiles = (int)((a.M + tile_m - 1) / tile_m);
  p.n_tiles = (int)((a.N + L->tbn - 1) / L->tbn);
  p.num_tiles = p.m_tiles * p.n_tiles;
  p.tiles_per_batch = p.num_tiles;
  p.group = L->pair ? pair_band_tiles(a.K) : GROUP_M;
  p.nk = (int)((a.K + BK - 1) / BK);
  p.act_scale = a.act_scale;
  p.per_token = a.act_per_token;
  p.w_scale = a.w_scale;
  p.bias = a.bias;
  p.y = a.y;
  p.acc = a.acc_out;
  p.y_elems = a.M * a.N;
  p.status = sw;
  L->grid = L->pair ? sm_count() / 2 : sm_count();
  if (L->grid > p.num_tiles) L->grid = p.num_tiles;
  return true;
}
}  // namespace

sq_status launch_gemm(const GemmArgs& a, cudaStream_t st) {
  unsigned int* sw = status_word();
  if (!sw) return fail(SQ_ERR_CUDA, "sq_gemm_w8a8: device status word unavailable");
  if (use_small(a.M, a.N)) {
    SmallParams p{};
    p.M = (int)a.M; p.N = (int)a.N; p.K = (int)a.K;
    p.n_tiles = (int)((a.N + SM_BM - 1) / SM_BM);
    p.nk = (int)((a.K + BK - 1) / BK);
    p.units = (int64_t)p.n_tiles * p.nk;
    p.grid = (int)small_grid(a.N, a.K);
    p.act_scale = a.act_scale;
    p.per_token = a.act_per_token;
    p.w_scale = a.w_scale;
    p.bias = a.bias;
    p.y = a.y;
    p.acc = a.acc_out;
    p.counters = reinterpret_cast<unsigned int*>(a.workspace);
    p.slots = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(a.workspace) +
                                         counters_bytes(a.N));
    p.status = sw;
    cudaError_t e = cudaMemsetAsync(a.workspace, 0, counters_bytes(a.N), st);
    if (e == cudaSuccess)
      e = a.yt == SQ_BF16 ? launch_small<true>(a, p, st) : launch_small<false>(a, p, st);
    if (e != cudaSuccess) return fail(SQ_ERR_CUDA, "sq_gemm_w8a8: %s", cudaGetErrorString(e));
    return SQ_OK;
  }
  LargeSetup L;
  if (!setup_large(a, sw, &L, true))
    return fail(SQ_ERR_CUDA, "sq_gemm_w8a8: cuTensorMapEncodeTiled failed");
  // TMA stores need 16-byte row pitches; other widths store directly
  const bool bf16 = a.yt == SQ_BF16;
  L.p.tma_store = (a.N % (bf16 ? 8 : 4)) == 0 &&
                  make_tmap_out(&L.ty, a.y, (uint64_t)a.N, (uint64_t)a.M, bf16);
  cudaError_t e;
  if (L.pair) {
    if (L.tbn == 256)
      e = bf16 ? launch_tc_pair<true, 256>(L.ta, L.tb, L.ty, L.p, L.grid, st)
               : launch_tc_pair<false, 256>(L.ta, L.tb, L.ty, L.p, L.grid, st);
    else
      e = bf16 ? launch_tc_pair<true, 192>(L.ta, L.tb, L.ty, L.p, L.grid, st)
               : launch_tc_pair<false, 192>(L.ta, L.tb, L.ty, L.p, L.grid, st);
  } else {
    e = launch_tiles<false>(L.ta, L.tb, L.ty, L.p, L.grid, L.tbn, bf16, st);
  }
  if (e != cudaSuccess) return fail(SQ_ERR_CUDA, "sq_gemm_w8a8: %s", cudaGetErrorString(e));
  return SQ_OK;
}

bool gemm_err_ok(int64_t M, int64_t N) { return M > 0 && N > 0 && !use_small(M, N); }

int gemm_err_max_slots() { return 12 * sm_count(); }

sq_status launch_gemm_err(const GemmArgs& a, const float* y_ref, double* part, int* nslots,
                          cudaStream_t st) {
  unsigned int* sw = status_word();
  if (!sw) return fail(SQ_ERR_CUDA, "sq_alpha_sweep: device status word unavailable");
  if (!gemm_err_ok(a.M, a.N)) return fail(SQ_ERR_UNSUPPORTED, "sq_alpha_sweep: error-mode GEMM shape");
  LargeSetup L;
  if (!setup_large(a, sw, &L, false))
    return fail(SQ_ERR_CUDA, "sq_alpha_sweep: cuTensorMapEncodeTiled failed");
  L.p.tma_store = 0;  // nothing is stored
  L.p.err_ref = y_ref;
  L.p.err_part = part;
  // twelve epilogue warps at any K: the epilogue reads y_ref and sums in
  // fp64, which one warp per TMEM quarter cannot hide behind the main loop
  // (measured on 2048 x 12288 x 4096: 177 -> 143 us per alpha of the sweep)
  const cudaError_t e =
      L.tbn == 256 ? launch_tc<false, 256, false, 2, 12, true>(L.ta, L.tb, L.ty, L.p, L.grid, st)
                   : launch_tc<false, 192, false, 2, 12, true>(L.ta, L.tb, L.ty, L.p, L.grid, st);
  if (e != cudaSuccess) return fail(SQ_ERR_CUDA, "sq_alpha_sweep: %s", cudaGetErrorString(e));
  *nslots = L.grid * 12;
  return SQ_OK;
}

sq_status launch_bmm(const BmmArgs& a, cudaStream_t st) {
  unsigned int* sw = status_word();
  if (!sw) return fail(SQ_ERR_CUDA, "sq_bmm_w8a8: device status word unavailable");
  const int sms = sm_count();
  const int tbn = pick_tile_n(a.M, a.N, sms, a.batch, true);
  CUtensorMap ta, tb;
  if (!make_tmap3(&ta, a.xq, (uint64_t)a.K, (uint64_t)a.M, (uint64_t)a.batch, BM) ||
      !make_tmap3(&tb, a.wq, (uint64_t)a.K, (uint64_t)a.N, (uint64_t)a.batch, (uint32_t)tbn))
    return fail(SQ_ERR_CUDA, "sq_bmm_w8a8: cuTensorMapEncodeTiled failed");
  Params p{};
  p.M = (int)a.M; p.N = (int)a.N; p.K = (int)a.K;
  p.m_tiles = (int)((a.M + BM - 1) / BM);
  p.n_tiles = (int)((a.N + tbn - 1) / tbn);
  p.tiles_per_batch = p.m_tiles * p.n_tiles;
  p.num_tiles = (int)(a.batch * p.tiles_per_batch);
  p.group = GROUP_M;
  p.nk = (int)((a.K + BK - 1) / BK);
  p.w_per_tensor = a.w_per_channel ? 0 : 1;
  p.act_scale = a.act_scale;
  p.per_token = a.act_per_token;
  p.w_scale = a.w_scale;
  p.bias = nullptr;
  p.y = a.y;
  p.acc = a.acc_out;
  p.y_elems = a.batch * a.M * a.N;
  p.status = sw;
  CUtensorMap ty;
  memset(&ty, 0, sizeof ty);
  const bool bf16 = a.yt == SQ_BF16;
  p.tma_store = (a.N % (bf16 ? 8 : 4)) == 0 &&
                make_tmap_out3(&ty, a.y, (uint64_t)a.N, (uint64_t)a.M, (uint64_t)a.batch, bf16);
  int grid = sms;
  if (grid > p.num_tiles) grid = p.num_tiles;
  const cudaError_t e = launch_tiles<true>(ta, tb, ty, p, grid, tbn, bf16, st);
  if (e != cudaSuccess) return fail(SQ_ERR_CUDA, "sq_bmm_w8a8: %s", cudaGetErrorString(e));
  return SQ_OK;
}

}  // namespace sq
