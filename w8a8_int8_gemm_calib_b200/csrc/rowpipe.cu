// rowpipe.cu -- the row-wise HBM-bound steps of the smoothed W8A8 linear
// layer as a TMA bulk-copy pipeline on sm_100a: the LayerNorm-fused
// calibration peak, the per-output-channel weight quantizer (W * s), and the
// runtime fused LayerNorm + smoothing + symmetric INT8 activation quantizer.
//
// Sources:
//   [review]   "SmoothQuant：大型语言模型的精准高效训练后量化 — 深度技术评审"
//              §2.2 (symmetric quantizer, step max|X|/127, round to nearest),
//              §2.5-2.6 (static per-tensor / dynamic per-token steps), §5.5
//   [embedded] "嵌入式 SLM 动态权重量化：SmoothQuant 激活异常值迁移与 INT8 部署实战"
//              §二 (modified LayerNorm with gamma/s, beta/s feeding the INT8
//              quantizer; W * diag(s) with static per-channel INT8)
//
// Design.  One CTA per SM: a producer warp streams whole rows (contiguous
// K-element runs) from HBM into a ring of up to 24 shared-memory row slots
// with 1-D bulk copies completing on mbarriers; slices of W warps consume the
// rows.  A thread loads its part of a row into registers as fp32 at once and
// hands the slot back, then works on the registers in place (x, x - mu, y).
// The slice emulates the 128 canonical LayerNorm slots, which fixes the
// reduction order (see rowops.cu; both files implement the same order).
// Per-column parameters (gamma, beta, or the column multiplier) are staged in
// shared memory once per CTA.  Every mbarrier wait is bounded.
//
// Rounding: r = y * (1/Delta) is clamped to [-127, 127] (NaN -> 0) and
// 1.5 * 2^23 is added: the fp32 addition rounds r to the nearest integer, ties
// to even, and the low byte of the sum's bit pattern is the two's-complement
// code (the constant's low byte is zero).  This equals round-half-even then
// clamp, without the quarter-rate float-to-int conversion.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "launch.cuh"
#include "sq_device.cuh"
#include "sq_internal.h"
#include "tc_ptx.cuh"

namespace sq {

namespace {

constexpr int kConsumers = 512;        // consumer threads per CTA
constexpr int kThreads = kConsumers + 32;
constexpr int kMaxSlots = 24;
constexpr size_t kSmemBudget = 226 * 1024;  // + static shared memory stays under the 227 KB per-block limit
constexpr size_t kSmemBudget2 = 112 * 1024;  // two CTAs per SM (228 KB per SM)
constexpr uint32_t kCopyPiece = 32768;
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr uint64_t kDrainNs = 1000000000ull;
constexpr int kSrcSmem = 0, kSrcRaw = 1, kSrcF32 = 2;

struct Pipe {
  RowArgs a;
  int64_t rows_per_cta;
  uint32_t row_bytes;
  int slots;
  int count;  // accumulate n_clipped
  unsigned int* status;
};

template <int ST>
__device__ __forceinline__ void slice_sync_t(int q) {
  asm volatile("bar.sync %0, %1;" ::"r"(q + 1), "r"(ST) : "memory");
}
// slice-wide AND of v (also a barrier of the slice)
template <int ST>
__device__ __forceinline__ bool slice_and_t(int q, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, o;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred o, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, o;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(q + 1), "r"(ST)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ float bsum(float p) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) p = __fadd_rn(p, __shfl_xor_sync(0xffffffffu, p, o));
  return p;
}
__device__ __forceinline__ float bmax(float p) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) p = fmaxf(p, __shfl_xor_sync(0xffffffffu, p, o));
  return p;
}

// One chunk of a row in shared memory, in storage form (8 bf16 or 8 fp32).
template <typename T> struct RawC;
template <> struct RawC<uint16_t> { uint4 a; };
template <> struct RawC<float> { uint4 a, b; };

__device__ __forceinline__ void lds_raw(const uint8_t* row, int c, RawC<uint16_t>& r) {
  r.a = *reinterpret_cast<const uint4*>(row + c * 16);
}
__device__ __forceinline__ void lds_raw(const uint8_t* row, int c, RawC<float>& r) {
  r.a = *reinterpret_cast<const uint4*>(row + c * 32);
  r.b = *reinterpret_cast<const uint4*>(row + c * 32 + 16);
}
// a chunk as four (even, odd) element pairs
__device__ __forceinline__ void unpack8(const RawC<uint16_t>& r, float2 (&v)[4]) {
  v[0] = make_float2(bf16lo(r.a.x), bf16hi(r.a.x));
  v[1] = make_float2(bf16lo(r.a.y), bf16hi(r.a.y));
  v[2] = make_float2(bf16lo(r.a.z), bf16hi(r.a.z));
  v[3] = make_float2(bf16lo(r.a.w), bf16hi(r.a.w));
}
__device__ __forceinline__ void unpack8(const RawC<float>& r, float2 (&v)[4]) {
  v[0] = make_float2(__uint_as_float(r.a.x), __uint_as_float(r.a.y));
  v[1] = make_float2(__uint_as_float(r.a.z), __uint_as_float(r.a.w));
  v[2] = make_float2(__uint_as_float(r.b.x), __uint_as_float(r.b.y));
  v[3] = make_float2(__uint_as_float(r.b.z), __uint_as_float(r.b.w));
}

// Per-column parameters live in shared memory in a split layout: elements
// 0-3 of chunk c at [4c, 4c+4), elements 4-7 at [K/2 + 4c, K/2 + 4c + 4).
// Lanes that read consecutive chunks then read consecutive 16-byte words
// (a 128-bit load per lane without bank conflicts).
__device__ __forceinline__ int param_index(int k, int half) {
  const int c = k >> 3, e = k & 7;
  return e < 4 ? c * 4 + e : half + c * 4 + (e - 4);
}
__device__ __forceinline__ void lds8(const float* p, int c, int half, float2 (&v)[4]) {
  const float4 a = *reinterpret_cast<const float4*>(p + c * 4);
  const float4 b = *reinterpret_cast<const float4*>(p + half + c * 4);
  v[0] = make_float2(a.x, a.y); v[1] = make_float2(a.z, a.w);
  v[2] = make_float2(b.x, b.y); v[3] = make_float2(b.z, b.w);
}

// Packed (even, odd) fp32 add and multiply, each lane one IEEE
// round-to-nearest operation.  They are used only where no multiply feeds an
// add: the code generator was seen to fuse a packed multiply and a following
// packed add into one fused multiply-add (one rounding instead of two) even
// with the explicit .rn modifier and -fmad=false.  Every add that follows a
// multiply is the scalar __fadd_rn, which is never fused.
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 pa, pb, pd;\n\t"
      "mov.b64 pa, {%2, %3};\n\t"
      "mov.b64 pb, {%4, %5};\n\t"
      "add.rn.f32x2 pd, pa, pb;\n\t"
      "mov.b64 {%0, %1}, pd;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 r;
  asm("{\n\t.reg .b64 pa, pb, pd;\n\t"
      "mov.b64 pa, {%2, %3};\n\t"
      "mov.b64 pb, {%4, %5};\n\t"
      "mul.rn.f32x2 pd, pa, pb;\n\t"
      "mov.b64 {%0, %1}, pd;\n\t}"
      : "=f"(r.x), "=f"(r.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

// Producer (one thread): streams rows r0 .. r0+R-1 of P.a.x into the ring,
// row i into slot i mod S, each slot refilled once its consumers released it
// (empty barrier).  On a time-out it lets every copy already issued land
// before returning, so the CTA never exits with a bulk copy in flight.
__device__ __forceinline__ void produce_rows(const Pipe& P, uint32_t ring_u32, uint64_t* bars,
                                             int64_t r0, int64_t R, volatile int* abort_flag) {
  const int S = P.slots;
  const uint32_t RB = P.row_bytes;
  auto full_bar = [&](int s) { return tc::smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return tc::smem_u32(bars + kMaxSlots + s); };
  uint32_t issued = 0, issued_par = 0;
  bool ok = true;
  const uint8_t* src = reinterpret_cast<const uint8_t*>(P.a.x) + r0 * (int64_t)RB;
  for (int64_t i = 0; i < R; ++i) {
    const int s = (int)(i % S);
    const int64_t u = i / S;
    if (u > 0 && !tc::mbar_wait(empty_bar(s), (uint32_t)((u - 1) & 1), abort_flag, kWaitNs,
                                P.status)) {
      ok = false;
      break;
    }
    tc::mbar_arrive_expect_tx(full_bar(s), RB);
    for (uint32_t off = 0; off < RB; off += kCopyPiece) {
      const uint32_t n = RB - off < kCopyPiece ? RB - off : kCopyPiece;
      // a copy outside x is skipped: its row's barrier then never completes
      // and the consumers give up at their bounded wait
      if (in_bounds((r0 + i) * (int64_t)RB + off, n, P.a.T * (int64_t)RB, P.status))
        tc::bulk_load(ring_u32 + (uint32_t)s * RB + off, src + i * (int64_t)RB + off, n, full_bar(s));
    }
    issued |= 1u << s;
    issued_par = (issued_par & ~(1u << s)) | ((uint32_t)(u & 1) << s);
  }
  if (!ok) {
    int never = 0;
    for (int s = 0; s < S; ++s)
      if (issued & (1u << s))
        tc::mbar_wait(full_bar(s), (issued_par >> s) & 1u, &never, kDrainNs, P.status);
  }
}

// Consumer threads stage the per-column parameters (gamma and beta, or the
// column multiplier) into the split layout, the global loads batched so that
// several are in flight per thread, and zero the per-CTA column peaks
// (colmax_s, when given).
template <bool LN>
__device__ __forceinline__ void stage_params(const RowArgs& a, float* pg, float* pb,
                                             unsigned int* colmax_s, int K, int tid) {
  constexpr int U = 8;
  const int khalf = K >> 1;
  const bool has_mul = !LN && a.mul != nullptr;
  for (int k0 = tid; k0 < K; k0 += U * kConsumers) {
    float gv[U], bv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = k0 + u * kConsumers;
      gv[u] = 0.0f;
      bv[u] = 0.0f;
      if (k < K) {
        if (LN) {
          gv[u] = __ldcg(a.g + k);
          if (a.b) bv[u] = __ldcg(a.b + k);
        } else if (has_mul) {
          gv[u] = __ldcg(a.mul + k);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int k = k0 + u * kConsumers;
      if (k < K) {
        const int pk = param_index(k, khalf);
        if (LN) {
          pg[pk] = gv[u];
          pb[pk] = bv[u];
        } else if (has_mul) {
          pg[pk] = gv[u];
        }
        if (colmax_s) colmax_s[k] = 0u;
      }
    }
  }
}

// Ring ownership: slice q consumes the CTA's rows i = q, q + NS, ... and row
// i sits in slot i mod S.  The host makes S a multiple of NS, so each slot
// is consumed by exactly one slice, in order: a slice waits on a slot only
// for the phase after the one it released itself, never two phases ahead
// (mbarrier parity cannot tell those apart).
//
// Slices of W warps (ST = 32*W threads).  A slice emulates the 128 canonical
// LayerNorm slots: thread (v, l) -- warp v of the slice, lane l -- walks the
// chunks c = 32*v + l + ST*i, i = 0, 1, ...; chunk i belongs to slot
// 32*(v + W*(i mod G)) + l with G = 4/W slot groups per thread, so each slot
// still accumulates its own chunks in increasing c.  The slot groups are
// then combined exactly as (r0 + r2) + (r1 + r3).
//
// Element-wise arithmetic runs on (even, odd) pairs with the packed fp32
// instructions (add2, mul2) where no multiply feeds an add: each lane is the
// same IEEE round-to-nearest operation as its scalar form; x - mu is
// computed as x + (-mu), which IEEE defines identically.  The running sums of the
// LayerNorm stay scalar (their order is fixed).
template <typename T, int W, int CM, bool LN, int MODE, int NB>
__global__ void __launch_bounds__(kThreads, NB) rowpipe_kernel(const Pipe P) {
  constexpr int ST = 32 * W;            // threads per slice
  constexpr int NS = kConsumers / ST;   // slices per CTA
  constexpr int G = W <= 4 ? 4 / W : 1;  // slot groups per thread (LayerNorm modes: W <= 4)
  static_assert(!LN || W == 1 || W == 2 || W == 4, "the LayerNorm order needs 1-, 2- or 4-warp slices");
  static_assert(MODE != ROW_COLMAX || LN, "raw column peaks use the column-strip kernel");
  // where the row is kept while a slice works on it: fp32 registers (at most
  // 64 per thread with one CTA per SM, 32 with two; the column peaks count
  // too when they are kept), the storage form in registers, or the
  // shared-memory slot itself
  constexpr int SRC = CM == 0 ? kSrcSmem
                      : CM * 8 * (MODE == ROW_COLMAX ? 2 : 1) <= 64 / NB ? kSrcF32 : kSrcRaw;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float red[NS][2][3][W];
  __shared__ int abort_s;

  const RowArgs& a = P.a;
  const int64_t K = a.K, nchunk = K >> 3;
  const int S = P.slots;
  const uint32_t RB = P.row_bytes;
  uint8_t* ring = smem;
  float* pg = reinterpret_cast<float*>(smem + (size_t)S * RB);  // gamma or multiplier [K]
  float* pb = pg + K;                                            // beta [K] (LN)
  unsigned int* colmax_s = reinterpret_cast<unsigned int*>(LN ? pb + K : pb);
  uint64_t* bars = reinterpret_cast<uint64_t*>(colmax_s + (MODE == ROW_COLMAX ? K : 0));
  const uint32_t ring_u32 = tc::smem_u32(ring);
  auto full_bar = [&](int s) { return tc::smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return tc::smem_u32(bars + kMaxSlots + s); };

  const int tid = threadIdx.x;
  pdl_launch_dependents();
  const bool has_mul = !LN && a.mul != nullptr;
  const int khalf = (int)(K >> 1);
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      tc::mbar_init(full_bar(s), 1);
      tc::mbar_init(empty_bar(s), W);  // one arrival per consumer warp of the slice
    }
    abort_s = 0;
    tc::mbar_fence_init();
  }
  __syncthreads();
  pdl_wait();
  volatile int* abort_flag = &abort_s;

  const int64_t r0 = (int64_t)blockIdx.x * P.rows_per_cta;
  int64_t R = a.T - r0;
  if (R > P.rows_per_cta) R = P.rows_per_cta;
  if (R < 0) R = 0;
  unsigned clipped = 0;

  if (tid >= kConsumers) {
    if (tid == kConsumers) produce_rows(P, ring_u32, bars, r0, R, abort_flag);
  } else {
    // ------------------------------------------------------------ consumers
    stage_params<LN>(a, pg, pb, MODE == ROW_COLMAX ? colmax_s : nullptr, (int)K, tid);
    if constexpr (!LN)
      fold_columns(a.mul, a.fold_g, a.fold_b, a.fold_g_out, a.fold_b_out, K, tid, kConsumers);
    asm volatile("bar.sync 9, %0;" ::"r"(kConsumers) : "memory");  // consumers only

    const int q = tid / ST, j = tid % ST;
    const int v = j >> 5, lane = j & 31;
    const float kf = (float)K;
    // a LayerNorm subtracts the mean; an RMSNorm has none (x - 0 = x, the
    // shift is left out)
    const bool shift = LN && !a.rms;
    const bool has_beta = LN && a.b != nullptr;
    // x / K for a power-of-two K is x * (1/K) exactly (both are the correctly
    // rounded value of the same exact quotient): a multiply instead of a
    // division subroutine
    const bool k_pow2 = (K & (K - 1)) == 0;
    const float kinv = 1.0f / kf;
    auto divk = [&](float v) { return k_pow2 ? __fmul_rn(v, kinv) : __fdiv_rn(v, kf); };
    constexpr int NC = (MODE == ROW_COLMAX && CM > 0) ? CM * 8 : 1;
    float cmax[NC];
#pragma unroll
    for (int i = 0; i < NC; ++i) cmax[i] = 0.0f;
    float pk[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // ROW_PEAK: running max of |y| (NaN skipped)
    const float static_inv = MODE == ROW_STATIC ? __fdiv_rn(1.0f, __ldcg(a.scale)) : 0.0f;
    const bool count = P.count != 0;
    int parity = 0;
    const int nch = (int)nchunk;  // < 2^14 here: rows fit in shared memory
    auto chunk_of = [&](int i) -> int { return 32 * v + lane + ST * i; };
    auto sync = [&]() {
      if constexpr (W == 1) __syncwarp();
      else slice_sync_t<ST>(q);
    };

    for (int64_t i = q; i < R; i += NS) {
      const int s = (int)(i % S);
      const int64_t u = i / S;
      const bool ok = tc::mbar_wait(full_bar(s), (uint32_t)(u & 1), abort_flag, kWaitNs, P.status);
      if constexpr (W == 1) {
        if (!__all_sync(0xffffffffu, ok)) break;
      } else {
        if (!slice_and_t<ST>(q, ok)) break;
      }
      const uint8_t* rowp = ring + (size_t)s * RB;
      const int64_t row = r0 + i;

      // The thread's part of the row in registers: as fp32 pairs (updated in
      // place by the passes below: x, then x - mu, then y) or in storage form.
      float2 xf[SRC == kSrcF32 ? CM : 1][4];
      RawC<T> xr[SRC == kSrcRaw ? CM : 1];
      if constexpr (SRC != kSrcSmem) {
#pragma unroll
        for (int m = 0; m < CM; ++m) {
          const int c = chunk_of(m);
          if (c < nch) {
            if constexpr (SRC == kSrcF32) {
              RawC<T> r;
              lds_raw(rowp, c, r);
              unpack8(r, xf[m]);
            } else {
              lds_raw(rowp, c, xr[m]);
            }
          }
        }
        // the row now lives in registers: each warp hands the slot back at
        // once, so the producer refills it while this row is processed
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(empty_bar(s));
      }

      float2 negmu2 = make_float2(0.0f, 0.0f), rstd2 = make_float2(0.0f, 0.0f);
      // y of one chunk in place: ((x - mu) * rstd) * g + b from x - mu, or
      // x * m, or x.  Without a beta (RMSNorm, or a LayerNorm given none) the
      // addition of +0 is left out: it could only turn a -0 into +0, which
      // changes no peak and no code.
      auto ytrans = [&](int c, float2 (&x)[4]) {
        if constexpr (LN) {
          float2 g8[4];
          lds8(pg, c, khalf, g8);
          if (has_beta) {
            float2 b8[4];
            lds8(pb, c, khalf, b8);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 t = mul2(mul2(x[e], rstd2), g8[e]);
              x[e] = make_float2(__fadd_rn(t.x, b8[e].x), __fadd_rn(t.y, b8[e].y));
            }
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) x[e] = mul2(mul2(x[e], rstd2), g8[e]);
          }
        } else {
          if (has_mul) {
            float2 m8[4];
            lds8(pg, c, khalf, m8);
#pragma unroll
            for (int e = 0; e < 4; ++e) x[e] = mul2(x[e], m8[e]);
          }
        }
      };
      // f(m, c, x[4]) over the thread's chunks in increasing c, with x at
      // level `lvl` (0: x, 1: x - mu, 2: y).  The fp32 register copy is
      // already at the level the previous pass left it at; the other sources
      // recompute the level from the stored row.
      auto for_level = [&](int lvl, auto&& f) {
        auto lift = [&](int c, float2 (&x)[4]) {
          if (LN && lvl >= 1 && shift) {
#pragma unroll
            for (int e = 0; e < 4; ++e) x[e] = add2(x[e], negmu2);
          }
          if (lvl >= 2) ytrans(c, x);
        };
        if constexpr (SRC == kSrcF32) {
#pragma unroll
          for (int m = 0; m < CM; ++m) {
            const int c = chunk_of(m);
            if (c < nch) f(m, c, xf[m]);
          }
        } else if constexpr (SRC == kSrcRaw) {
#pragma unroll
          for (int m = 0; m < CM; ++m) {
            const int c = chunk_of(m);
            if (c < nch) {
              float2 x[4];
              unpack8(xr[m], x);
              lift(c, x);
              f(m, c, x);
            }
          }
        } else {
          int m = 0;
          for (int c = chunk_of(0); c < nch; c += ST, ++m) {
            RawC<T> r;
            lds_raw(rowp, c, r);
            float2 x[4];
            unpack8(r, x);
            lift(c, x);
            f(m, c, x);
          }
        }
      };
      // exact (r0 + r2) + (r1 + r3) of the per-slot partial sums p[g]
      auto slot_sum = [&](const float (&p)[G], int which) -> float {
        float t[G];
#pragma unroll
        for (int g = 0; g < G; ++g) t[g] = bsum(p[g]);
        if constexpr (W == 1) {  // one lane holds all four slot groups
          return __fadd_rn(__fadd_rn(t[0], t[2]), __fadd_rn(t[1], t[3]));
        }
        float mine = t[0];
        if constexpr (G == 2) mine = __fadd_rn(t[0], t[1]);  // r_v + r_(v+2)
        if (lane == 0) red[q][parity][which][v] = mine;
        sync();
        const float* r = red[q][parity][which];
        if constexpr (W == 4) return __fadd_rn(__fadd_rn(r[0], r[2]), __fadd_rn(r[1], r[3]));
        else return __fadd_rn(r[0], r[1]);
      };

      if constexpr (LN) {
        float p[G];
        // RMSNorm has no mean: mu = 0 makes x - mu = x below, the variance
        // pass the mean of squares, and y = ((x * rstd) * g) + 0 (beta NULL)
        float mu = 0.0f;
        if (!a.rms) {
#pragma unroll
          for (int g = 0; g < G; ++g) p[g] = 0.0f;
          for_level(0, [&](int m, int, float2 (&x)[4]) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              p[m % G] = __fadd_rn(p[m % G], x[e].x);
              p[m % G] = __fadd_rn(p[m % G], x[e].y);
            }
          });
          mu = divk(slot_sum(p, 0));
        }
        negmu2 = make_float2(-mu, -mu);
#pragma unroll
        for (int g = 0; g < G; ++g) p[g] = 0.0f;
        for_level(0, [&](int m, int, float2 (&x)[4]) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (shift) x[e] = add2(x[e], negmu2);  // now x - mu
            p[m % G] = __fmaf_rn(x[e].x, x[e].x, p[m % G]);
            p[m % G] = __fmaf_rn(x[e].y, x[e].y, p[m % G]);
          }
        });
        const float rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(divk(slot_sum(p, 1)), a.eps)));
        rstd2 = make_float2(rstd, rstd);
      }
      constexpr int kLvlIn = LN ? 1 : 0;  // level the y pass starts from

      if constexpr (MODE == ROW_COLMAX) {
        for_level(kLvlIn, [&](int m, int c, float2 (&x)[4]) {
          ytrans(c, x);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if constexpr (CM > 0) {
              cmax[m * 8 + 2 * e] = fmaxf(cmax[m * 8 + 2 * e], fabsf(x[e].x));
              cmax[m * 8 + 2 * e + 1] = fmaxf(cmax[m * 8 + 2 * e + 1], fabsf(x[e].y));
            } else {
              atomicMax(&colmax_s[c * 8 + 2 * e], peak_bits(fabsf(x[e].x)));
              atomicMax(&colmax_s[c * 8 + 2 * e + 1], peak_bits(fabsf(x[e].y)));
            }
          }
        });
      } else if constexpr (MODE == ROW_PEAK) {
        for_level(kLvlIn, [&](int, int c, float2 (&x)[4]) {
          ytrans(c, x);
#pragma unroll
          for (int e = 0; e < 4; ++e) pk[e] = fmaxf(fmaxf(pk[e], fabsf(x[e].x)), fabsf(x[e].y));
        });
      } else if constexpr (MODE == ROW_STATIC) {
        int8_t* qr = a.q + row * K;
        for_level(kLvlIn, [&](int, int c, float2 (&x)[4]) {
          ytrans(c, x);
          uint32_t b[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            b[2 * e] = qbits(x[e].x, static_inv, count, clipped);
            b[2 * e + 1] = qbits(x[e].y, static_inv, count, clipped);
          }
          if (in_bounds(row * K + c * 8, 8, a.T * K, P.status)) store_codes(qr + c * 8, b);
        });
      } else {
        // peak magnitude with NaN propagated: a finite result means every
        // element is finite (and then it equals the NaN-ignoring peak).  The
        // maximum is exact in any order: four independent chains per thread.
        float m4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        for_level(kLvlIn, [&](int, int c, float2 (&x)[4]) {
          ytrans(c, x);  // now y
#pragma unroll
          for (int e = 0; e < 4; ++e) m4[e] = max_nan3(m4[e], fabsf(x[e].x), fabsf(x[e].y));
        });
        float mn = warp_maxabs_nan(max_nan(max_nan3(m4[0], m4[1], m4[2]), m4[3]));
        if constexpr (W > 1) {
          if (lane == 0) red[q][parity][2][v] = mn;
          sync();
#pragma unroll
          for (int t = 0; t < W; ++t) mn = max_nan(mn, red[q][parity][2][t]);
        }
        float mx = mn;  // >= 0, or NaN
        const bool clean = mx < INFINITY;  // false for inf and NaN
        if (!clean) {
          // non-finite elements: the peak over the non-NaN values (fmaxf)
          float m2 = 0.0f;
          for_level(2, [&](int, int, float2 (&y)[4]) {
#pragma unroll
            for (int e = 0; e < 4; ++e) m2 = fmaxf(fmaxf(m2, fabsf(y[e].x)), fabsf(y[e].y));
          });
          m2 = bmax(m2);
          if constexpr (W > 1) {
            sync();  // everyone has read red[..][2] above
            if (lane == 0) red[q][parity][2][v] = m2;
            sync();
#pragma unroll
            for (int t = 0; t < W; ++t) m2 = fmaxf(m2, red[q][parity][2][t]);
          }
          mx = m2;
        }
        const float delta = __fdiv_rn(fmaxf(mx, 1e-7f), 127.0f);
        const float inv = __fdiv_rn(1.0f, delta);
        if (j == 0 && in_bounds(row, 1, a.T, P.status)) a.scale[row] = delta;
        int8_t* qr = a.q + row * K;
        if (clean) {
          // |y * inv| <= 127*(1 + 2^-23) < 127.5 for every element of a
          // finite row: round (1.5 * 2^23 addition) without clamping
          const float2 inv2 = make_float2(inv, inv);
          for_level(2, [&](int, int c, float2 (&y)[4]) {
            uint32_t b[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 r = mul2(y[e], inv2);
              b[2 * e] = __float_as_uint(__fadd_rn(r.x, kRoundMagic));
              b[2 * e + 1] = __float_as_uint(__fadd_rn(r.y, kRoundMagic));
            }
            if (in_bounds(row * K + c * 8, 8, a.T * K, P.status)) store_codes(qr + c * 8, b);
          });
        } else {
          for_level(2, [&](int, int c, float2 (&y)[4]) {
            uint32_t b[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              b[2 * e] = qbits(y[e].x, inv, count, clipped);
              b[2 * e + 1] = qbits(y[e].y, inv, count, clipped);
            }
            if (in_bounds(row * K + c * 8, 8, a.T * K, P.status)) store_codes(qr + c * 8, b);
          });
        }
      }
      if constexpr (SRC == kSrcSmem) {
        __syncwarp();  // this warp is done with the slot
        if (lane == 0) tc::mbar_arrive(empty_bar(s));
      }
      parity ^= 1;
    }
    if constexpr (MODE == ROW_PEAK) {
      const float m = bmax(fmaxf(fmaxf(pk[0], pk[1]), fmaxf(pk[2], pk[3])));
      if (lane == 0) atomicMax(reinterpret_cast<unsigned int*>(a.peak), __float_as_uint(m));
    }
    if constexpr (MODE == ROW_COLMAX && CM > 0) {
#pragma unroll
      for (int m = 0; m < CM; ++m) {
        const int c = chunk_of(m);
        if (c < nch && R > 0) {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            atomicMax(&colmax_s[c * 8 + e], __float_as_uint(cmax[m * 8 + e]));
        }
      }
    }
  }
  __syncthreads();
  if constexpr (MODE == ROW_COLMAX) {
    if (tid < kConsumers && R > 0)
      for (int64_t k = tid; k < K; k += kConsumers)
        if (in_bounds(k, 1, K, P.status))
          atomicMax(reinterpret_cast<unsigned int*>(a.colmax) + k, colmax_s[k]);
  }
  if (P.count && tid < kConsumers) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) clipped += __shfl_xor_sync(0xffffffffu, clipped, o);
    if ((tid & 31) == 0 && clipped) atomicAdd(a.n_clipped, (unsigned long long)clipped);
  }
}

// Shared memory after the ring: parameters (gamma and beta, or the column
// multiplier: the region exists even when no multiplier is given), the
// per-CTA column peaks (column-peak mode), and the mbarriers.
size_t fixed_smem(int64_t K, bool ln, RowMode mode) {
  size_t b = (ln ? 2 : 1) * (size_t)K * 4;
  if (mode == ROW_COLMAX) b += (size_t)K * 4;
  return b + 2 * kMaxSlots * 8;
}

template <typename T, int W, int CM, bool LN, int MODE, int NB = 1>
cudaError_t launch_t(const Pipe& P, size_t smem, int grid, cudaStream_t st) {
  auto kern = rowpipe_kernel<T, W, CM, LN, MODE, NB>;
  // the shared-memory limit is raised once per instantiation (and per
  // device), to the whole budget, so that launches stay free of driver calls
  static std::once_flag once[64];
  static cudaError_t attr_err[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= 64) return e != cudaSuccess ? e : cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] {
    attr_err[dev] = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(NB == 2 ? kSmemBudget2 : kSmemBudget));
  });
  if (attr_err[dev] != cudaSuccess) return attr_err[dev];
  return launch_pdl(kern, dim3(grid), dim3(kThreads), smem, st, P);
}

// Quantizing modes.  The host picks the slice width W (warps): the narrowest
// whose threads hold at most 8 chunks each -- the row then sits in fp32
// registers, worked on in place -- while every slice has a slot (W = 1 gives
// 16 slices and reductions by warp shuffles alone; a LayerNorm's fixed
// reduction order allows W <= 4).  Up to 16 bf16 chunks per thread are held
// in storage form instead; beyond that each pass re-reads shared memory.
template <typename T, int W, bool LN, int MODE>
cudaError_t dispatch_quant_w(const Pipe& P, int nb, size_t smem, int grid, cudaStream_t st) {
  constexpr bool kBf16 = sizeof(T) == 2;
  const int64_t per = (P.a.K / 8 + 32 * W - 1) / (32 * W);
  if constexpr (!LN && W >= 2 && W <= 4) {
    if (nb == 2) {  // two CTAs per SM: at most 4 chunks per thread
      if (per <= 2) return launch_t<T, W, 2, LN, MODE, 2>(P, smem, grid, st);
      if (per <= 4) return launch_t<T, W, 4, LN, MODE, 2>(P, smem, grid, st);
      return cudaErrorInvalidValue;
    }
  }
  if (nb != 1) return cudaErrorInvalidValue;
  if (per <= 2) return launch_t<T, W, 2, LN, MODE>(P, smem, grid, st);
  if (per <= 4) return launch_t<T, W, 4, LN, MODE>(P, smem, grid, st);
  if (per <= 8) return launch_t<T, W, 8, LN, MODE>(P, smem, grid, st);
  if constexpr (kBf16) {
    if (per <= 16) return launch_t<T, W, 16, LN, MODE>(P, smem, grid, st);
  }
  return launch_t<T, W, 0, LN, MODE>(P, smem, grid, st);
}

template <typename T, bool LN, int MODE>
cudaError_t dispatch_quant(const Pipe& P, int w, int nb, size_t smem, int grid, cudaStream_t st) {
  if (w == 1) return dispatch_quant_w<T, 1, LN, MODE>(P, nb, smem, grid, st);
  if (w == 2) return dispatch_quant_w<T, 2, LN, MODE>(P, nb, smem, grid, st);
  if (w == 4) return dispatch_quant_w<T, 4, LN, MODE>(P, nb, smem, grid, st);
  if constexpr (!LN) {
    if (w == 8) return dispatch_quant_w<T, 8, LN, MODE>(P, nb, smem, grid, st);
    if (w == 16) return dispatch_quant_w<T, 16, LN, MODE>(P, nb, smem, grid, st);
  }
  return cudaErrorInvalidValue;
}

// Column-peak mode: 128-thread slices; the running peak of each owned
// element stays in registers for up to 4 chunks per thread (with the row in
// fp32) or 6 (bf16, the row in storage form).
template <typename T>
cudaError_t dispatch_colmax(const Pipe& P, size_t smem, int grid, cudaStream_t st) {
  const int64_t per = (P.a.K / 8 + 127) / 128;
  switch (per) {
    case 1: return launch_t<T, 4, 1, true, ROW_COLMAX>(P, smem, grid, st);
    case 2: return launch_t<T, 4, 2, true, ROW_COLMAX>(P, smem, grid, st);
    case 3: return launch_t<T, 4, 3, true, ROW_COLMAX>(P, smem, grid, st);
    case 4: return launch_t<T, 4, 4, true, ROW_COLMAX>(P, smem, grid, st);
    default: break;
  }
  if constexpr (sizeof(T) == 2) {  // bf16 rows held in storage form
    if (per == 5) return launch_t<T, 4, 5, true, ROW_COLMAX>(P, smem, grid, st);
    if (per == 6) return launch_t<T, 4, 6, true, ROW_COLMAX>(P, smem, grid, st);
  }
  return launch_t<T, 4, 0, true, ROW_COLMAX>(P, smem, grid, st);
}

template <typename T>
cudaError_t dispatch_mode(const Pipe& P, RowMode mode, int w, int nb, size_t smem, int grid,
                          cudaStream_t st) {
  const bool ln = P.a.g != nullptr;
  switch (mode) {
    case ROW_DYNAMIC:
      return ln ? dispatch_quant<T, true, ROW_DYNAMIC>(P, w, nb, smem, grid, st)
                : dispatch_quant<T, false, ROW_DYNAMIC>(P, w, nb, smem, grid, st);
    case ROW_STATIC:
      return ln ? dispatch_quant<T, true, ROW_STATIC>(P, w, nb, smem, grid, st)
                : dispatch_quant<T, false, ROW_STATIC>(P, w, nb, smem, grid, st);
    case ROW_PEAK:
      return ln ? dispatch_quant<T, true, ROW_PEAK>(P, w, nb, smem, grid, st)
                : dispatch_quant<T, false, ROW_PEAK>(P, w, nb, smem, grid, st);
    case ROW_COLMAX:
      return ln && nb == 1 ? dispatch_colmax<T>(P, smem, grid, st) : cudaErrorInvalidValue;
  }
  return cudaErrorInvalidValue;
}

// Ring depth, slice width and CTAs per SM: returns false when no valid
// combination fits.  `slots` is a multiple of the slice count 16/w.  Rows
// without a LayerNorm (the weight fold, the plain quantizer) run two CTAs
// per SM -- twice the resident warps -- when slices of at most 4 warps
// hold the row with at most 4 chunks per thread and each slice still gets
// two slots of look-ahead (measured: K = 4096 gains, wider rows, which
// would need 8-warp slices and 4 slots, lose); everything else runs one
// CTA per SM.
bool plan(int64_t K, sq_dtype xt, RowMode mode, bool ln, int* slots, int* w, int* nb,
          size_t* smem) {
  const size_t rb = (size_t)K * (xt == SQ_BF16 ? 2 : 4);
  const size_t fixed = fixed_smem(K, ln, mode);
  const int64_t nch = K / 8;
  if (mode == ROW_COLMAX && !ln) return false;  // raw peaks: column strips (rowops.cu)
  if (!ln && mode != ROW_COLMAX && fixed + 2 * rb <= kSmemBudget2) {
    int s2 = (int)((kSmemBudget2 - fixed) / rb);
    if (s2 > kMaxSlots) s2 = kMaxSlots;
    for (int c = 2; c <= 4; c *= 2) {
      const int ns = kConsumers / (32 * c);
      if ((nch + 32 * c - 1) / (32 * c) <= 4 && s2 >= 2 * ns) {
        *slots = (s2 / ns) * ns;
        *w = c;
        *nb = 2;
        *smem = (size_t)*slots * rb + fixed;
        return true;
      }
    }
  }
  if (fixed + 2 * rb > kSmemBudget) return false;
  int s = (int)((kSmemBudget - fixed) / rb);
  if (s > kMaxSlots) s = kMaxSlots;
  int ww = 0;
  if (mode == ROW_COLMAX) {
    ww = 4;
  } else {
    // the narrowest slice that holds its part of the row in fp32 registers
    // (at most 8 chunks per thread) and has a slot per slice
    for (int c = 1; c <= (ln ? 4 : 16); c *= 2)
      if ((nch + 32 * c - 1) / (32 * c) <= 8 && s >= kConsumers / (32 * c)) {
        ww = c;
        break;
      }
    if (ww == 0) {
      if (s >= 8) ww = 2;
      else if (s >= 4) ww = 4;
      else if (!ln) ww = 8;  // two slices of 8 warps share the (2 or 3) slots
      else return false;
    }
  }
  const int ns = kConsumers / (32 * ww);
  if (s < ns || s < 2) return false;
  s = (s / ns) * ns;
  *slots = s;
  *w = ww;
  *nb = 1;
  *smem = (size_t)s * rb + fixed;
  return true;
}

}  // namespace

bool rowpipe_fits(int64_t K, sq_dtype xt, RowMode mode, bool ln) {
  int slots, w, nb;
  size_t smem;
  return plan(K, xt, mode, ln, &slots, &w, &nb, &smem);
}

cudaError_t launch_rowpipe(const RowArgs& a, sq_dtype xt, RowMode mode, cudaStream_t st) {
  const size_t rb = (size_t)a.K * (xt == SQ_BF16 ? 2 : 4);
  int slots = 0, w = 0, nb = 1;
  size_t smem = 0;
  if (!plan(a.K, xt, mode, a.g != nullptr, &slots, &w, &nb, &smem)) return cudaErrorInvalidValue;
  unsigned int* sw = status_word();
  if (!sw) return cudaErrorInvalidDevice;
  int grid = sm_count() * nb;
  if ((int64_t)grid > a.T) grid = (int)a.T;
  Pipe P{};
  P.a = a;
  P.rows_per_cta = (a.T + grid - 1) / grid;
  grid = (int)((a.T + P.rows_per_cta - 1) / P.rows_per_cta);
  P.row_bytes = (uint32_t)rb;
  P.slots = slots;
  P.count = a.n_clipped != nullptr;
  P.status = sw;
  return xt == SQ_BF16 ? dispatch_mode<uint16_t>(P, mode, w, nb, smem, grid, st)
                       : dispatch_mode<float>(P, mode, w, nb, smem, grid, st);
}

}  // namespace sq
