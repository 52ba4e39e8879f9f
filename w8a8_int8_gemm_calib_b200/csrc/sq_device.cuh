// sq_device.cuh -- small device helpers shared by the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sq {

// Device status codes written to the status word (values of sq_status).
constexpr unsigned kStatusTimeout = 7u;
constexpr unsigned kStatusBounds = 9u;

__device__ __forceinline__ void set_status(unsigned int* status, unsigned code) {
  if (status) atomicCAS(status, 0u, code);
}

// Bounds check of a hand-computed global-memory offset: the access of
// elements [off, off + n) of a tensor of `size` elements may go ahead.  In
// a build with SQ_DEBUG_BOUNDS an offset outside records SQ_ERR_BOUNDS and
// the caller skips the access; otherwise the check is compiled away.
__device__ __forceinline__ bool in_bounds(int64_t off, int64_t n, int64_t size,
                                          unsigned int* status) {
#ifdef SQ_DEBUG_BOUNDS
  if (off < 0 || n < 0 || off + n > size) {
    set_status(status, kStatusBounds);
    return false;
  }
#else
  (void)off; (void)n; (void)size; (void)status;
#endif
  return true;
}

// bf16 -> fp32 is exact: the bf16 pattern is the upper half of the fp32 one.
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// One 8-element chunk of an fp32 or bf16 row, in its storage form.
template <typename T> struct Raw8;
template <> struct Raw8<float> { float4 a, b; };
template <> struct Raw8<uint16_t> { uint4 a; };

// Loads of data that an earlier kernel of the stream may have written.
// Every kernel here is launched with programmatic dependent launch: it may
// start while the kernels before it still run, and only its
// griddepcontrol.wait orders it after them.  The read-only (.nc) path and
// L1 are not kept coherent with those writes, so such data -- activations,
// 1/s, steps, folded parameters, weight scales -- is read at L2 (.cg).

// Streaming (read-once) loads, at L2.
__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 r;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

__device__ __forceinline__ void load_raw(const float* p, Raw8<float>& r) {
  uint4 a = ld_stream_u4(p), b = ld_stream_u4(p + 4);
  r.a = make_float4(__uint_as_float(a.x), __uint_as_float(a.y), __uint_as_float(a.z), __uint_as_float(a.w));
  r.b = make_float4(__uint_as_float(b.x), __uint_as_float(b.y), __uint_as_float(b.z), __uint_as_float(b.w));
}
__device__ __forceinline__ void load_raw(const uint16_t* p, Raw8<uint16_t>& r) {
  r.a = ld_stream_u4(p);
}

// Rows read more than once (also at L2).
__device__ __forceinline__ void load_raw_cached(const float* p, Raw8<float>& r) {
  r.a = __ldcg(reinterpret_cast<const float4*>(p));
  r.b = __ldcg(reinterpret_cast<const float4*>(p) + 1);
}
__device__ __forceinline__ void load_raw_cached(const uint16_t* p, Raw8<uint16_t>& r) {
  r.a = __ldcg(reinterpret_cast<const uint4*>(p));
}

__device__ __forceinline__ void unpack(const Raw8<float>& r, float (&v)[8]) {
  v[0] = r.a.x; v[1] = r.a.y; v[2] = r.a.z; v[3] = r.a.w;
  v[4] = r.b.x; v[5] = r.b.y; v[6] = r.b.z; v[7] = r.b.w;
}
__device__ __forceinline__ void unpack(const Raw8<uint16_t>& r, float (&v)[8]) {
  v[0] = bf16lo(r.a.x); v[1] = bf16hi(r.a.x);
  v[2] = bf16lo(r.a.y); v[3] = bf16hi(r.a.y);
  v[4] = bf16lo(r.a.z); v[5] = bf16hi(r.a.z);
  v[6] = bf16lo(r.a.w); v[7] = bf16hi(r.a.w);
}

// Q(y; Delta) given inv = 1/Delta, as the fp32 whose low byte is the code:
// r = y * inv is clamped to [-127, 127] (NaN -> 0) and 1.5 * 2^23 is added;
// the fp32 addition rounds r to the nearest integer, ties to even, and the
// low byte of the sum's bit pattern is the two's-complement code (the
// constant's low byte is zero).  This equals round-half-even then clamp,
// without the quarter-rate float-to-int conversion.  count: values that
// round outside [-127, 127] are counted in `clipped`.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
__device__ __forceinline__ uint32_t qbits(float y, float inv, bool count, unsigned& clipped) {
  float r = __fmul_rn(y, inv);
  if (count) clipped += fabsf(r) >= 127.5f;  // rounds outside [-127, 127]
  r = (r != r) ? 0.0f : r;
  r = fminf(fmaxf(r, -127.0f), 127.0f);
  return __float_as_uint(__fadd_rn(r, kRoundMagic));
}

// Low bytes of four qbits results, packed little-endian.
__device__ __forceinline__ uint32_t pack4u(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  const uint32_t lo = __byte_perm(a, b, 0x0040);
  const uint32_t hi = __byte_perm(c, d, 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}
__device__ __forceinline__ void store_codes(int8_t* dst, const uint32_t (&b)[8]) {
  uint2 pk;
  pk.x = pack4u(b[0], b[1], b[2], b[3]);
  pk.y = pack4u(b[4], b[5], b[6], b[7]);
  *reinterpret_cast<uint2*>(dst) = pk;
}

// The fp32 bit pattern of a magnitude |y| for an unsigned atomic max (the
// order of the patterns of non-negative floats is their numeric order); a
// NaN gives 0, so that column peaks skip NaN as fmaxf does.
__device__ __forceinline__ unsigned int peak_bits(float a) {
  return a != a ? 0u : __float_as_uint(a);
}

// Maxima with NaN propagated: NaN if any operand is NaN.  The three-operand
// form takes |a| and |b| as operand modifiers (one instruction for two
// elements); the warp form is one redux over the 32 lanes' magnitudes.
__device__ __forceinline__ float max_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float max_nan3(float a, float b, float c) {
  float r;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float warp_maxabs_nan(float v) {
  float r;
  asm volatile("redux.sync.max.abs.NaN.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// 8 consecutive fp32 parameters (gamma, beta, multipliers), at L2.
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  float4 a = __ldcg(reinterpret_cast<const float4*>(p));
  float4 b = __ldcg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Q(y; Delta) given 1/Delta: round half to even (cvt.rni: NaN -> 0,
// +-inf -> saturated), then clamp to the symmetric range [-127, 127].
__device__ __forceinline__ int quant_code(float y, float inv, unsigned& clipped) {
  int q = __float2int_rn(__fmul_rn(y, inv));
  clipped += (q > 127) | (q < -127);
  return max(-127, min(127, q));
}

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  uint32_t lo = __byte_perm((uint32_t)a, (uint32_t)b, 0x0040);  // a.b0, b.b0 -> bytes 0,1
  uint32_t hi = __byte_perm((uint32_t)c, (uint32_t)d, 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

// g_out = g / s and b_out = b / s over columns [0, K) (either output may be
// NULL), this CTA's share with nt threads: the LayerNorm fold that rides
// along with the weight fold, one IEEE fp32 division per element.
__device__ __forceinline__ void fold_columns(const float* s, const float* g, const float* b,
                                             float* g_out, float* b_out, int64_t K, int t,
                                             int nt) {
  if (!g_out && !b_out) return;
  for (int64_t k = (int64_t)blockIdx.x * nt + t; k < K; k += (int64_t)gridDim.x * nt) {
    const float sk = __ldcg(s + k);
    if (g_out) g_out[k] = __fdiv_rn(__ldcg(g + k), sk);
    if (b_out) b_out[k] = __fdiv_rn(__ldcg(b + k), sk);
  }
}

// Bounded-wait clock: nanoseconds from the global timer.
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Programmatic dependent launch.  Every kernel of this library is launched
// with programmatic stream serialization (launch_pdl, launch.cuh): it lets
// the next kernel of the stream begin launching at once (that kernel's
// blocks take SMs as they free up and run their data-free prologue), and it
// waits for the previous kernel of the stream to complete -- with its
// memory writes visible -- before its own first global-memory access.  Every
// thread of every block executes pdl_wait() before touching global memory
// and before it can exit, so completion stays transitive along the stream.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

}  // namespace sq
