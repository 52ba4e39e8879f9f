// sq_internal.h -- declarations shared by the C-ABI layer (api.cpp) and the
// kernel translation units.  Not part of the public interface (include/sq.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sq.h"

namespace sq {

// Zero `bytes` (a multiple of 4) at p with a kernel launched like every
// other one of this library (programmatic dependent launch), so that the
// kernel after it can overlap its launch, which a memset node prevents.
// Measured faster only where the next kernel is a short pass (the
// per-tensor step's reset); ahead of the weight column peaks a memset
// measured faster, so those keep it.
cudaError_t launch_zero(void* p, size_t bytes, cudaStream_t st);

// Device address of the per-device status word (a static __device__
// variable in status.cu), looked up once per device.  NULL on failure.
unsigned int* status_word();

// Number of SMs of the current device (cached per device).
int sm_count();

// Record a one-line host-side error for sq_last_error() and return `st`.
sq_status fail(sq_status st, const char* fmt, ...);

// ---------------------------------------------------------------- row ops
// Column absmax: out[k] = max(out[k], max_t |x[t,k]|) (out as fp32 bits,
// atomic max).  K % 8 == 0.
cudaError_t launch_colmax(const void* x, sq_dtype xt, int64_t T, int64_t K,
                          float* out, cudaStream_t st);

// ROW_PEAK: no codes; the peak of |y| over every row of the call is folded
// into *peak (per-tensor dynamic quantization, first pass).
enum RowMode { ROW_DYNAMIC = 0, ROW_STATIC = 1, ROW_COLMAX = 2, ROW_PEAK = 3 };

struct RowArgs {
  const void* x;
  int64_t T, K;
  const float* g;      // LayerNorm gamma (NULL: no LayerNorm)
  const float* b;      // LayerNorm beta (may be NULL)
  float eps;
  int rms;             // with g: RMSNorm (no mean; b must be NULL) instead of LayerNorm
  const float* mul;    // per-column multiplier when there is no LayerNorm (may be NULL)
  float* scale;        // ROW_DYNAMIC: out [T]; ROW_STATIC: in [1]
  int8_t* q;           // [T,K] codes out (quantizing modes)
  unsigned long long* n_clipped;  // may be NULL
  float* colmax;       // ROW_COLMAX: running max [K] (fp32 bits, atomic max)
  float* peak;         // ROW_PEAK: running peak [1] (fp32 bits, atomic max)
  // With mul (the weight fold): also fold_g_out = fold_g / mul and
  // fold_b_out = fold_b / mul over the K columns, shared out among the
  // launch's CTAs (each output NULL to skip it)
  const float* fold_g;
  const float* fold_b;
  float* fold_g_out;
  float* fold_b_out;
  unsigned int* status;  // the device status word (set by launch_row)
};

cudaError_t launch_row(const RowArgs& a, sq_dtype xt, RowMode mode,
                       cudaStream_t st);

// Rows held in registers (rowreg.cu): the static quantizer of bf16 rows
// without a LayerNorm, up to 20480 columns.
bool rowreg_fits(int64_t K, sq_dtype xt, RowMode mode, bool ln);
cudaError_t launch_rowreg(const RowArgs& a, RowMode mode, cudaStream_t st);

// Bulk-copy pipelined variant (rowpipe.cu), used whenever two row slots and
// the per-column parameters fit in shared memory.
bool rowpipe_fits(int64_t K, sq_dtype xt, RowMode mode, bool ln);
cudaError_t launch_rowpipe(const RowArgs& a, sq_dtype xt, RowMode mode,
                           cudaStream_t st);

// s / inv_s (and the static step) from amax_x and the weight column peaks
// amax_w (which may be s itself).
cudaError_t launch_scales(const float* amax_x, const float* amax_w, int64_t K, float alpha,
                          float* s, float* inv_s, float* delta_out, cudaStream_t st);

// act_scale[0] = Delta(act_scale[0]) = max(peak, 1e-7) / 127 (one thread).
cudaError_t launch_peak_to_delta(float* act_scale, cudaStream_t st);

// w_scale[k] /= s[k], bias[k] /= s[k] (bias may be NULL).
cudaError_t launch_fold_producer(const float* s, int64_t K, float* w_scale, float* bias,
                                 cudaStream_t st);

// Relative Frobenius error of y against y_ref (n fp32 values each), in
// fp64 and deterministic: *err = sqrt(sum (y - r)^2 / sum r^2) (0 / 0 = 0,
// x / 0 = inf).  scratch: output_error_scratch_bytes() of device memory.
size_t output_error_scratch_bytes();
cudaError_t launch_output_error(const float* y, const float* y_ref, int64_t n, double* scratch,
                                double* err, cudaStream_t st);
// The last step alone: *err from nslots (sum (y - r)^2, sum r^2) pairs.
cudaError_t launch_output_error_final(const double* part, int nslots, double* err,
                                      cudaStream_t st);

cudaError_t launch_fold_ln(const float* gamma, const float* beta,
                           const float* s, int64_t K, float* gamma_out,
                           float* beta_out, cudaStream_t st);

// ---------------------------------------------------------------- GEMM
struct GemmArgs {
  const int8_t* xq;
  const int8_t* wq;
  int64_t M, N, K;
  const float* act_scale;
  int act_per_token;
  const float* w_scale;
  const float* bias;  // [N] or NULL
  void* y;
  sq_dtype yt;
  int32_t* acc_out;
  void* workspace;
  size_t workspace_bytes;
};

// Batched INT8 GEMM (attention BMMs): y[b] = xq[b] wq[b]^T dequantized
// per batch; act_scale [batch*M] (per token) or [batch]; w_scale [batch*N]
// (per channel) or [batch]; y, acc_out [batch, M, N].
struct BmmArgs {
  const int8_t* xq;
  const int8_t* wq;
  int64_t batch, M, N, K;
  const float* act_scale;
  int act_per_token;
  const float* w_scale;
  int w_per_channel;
  void* y;
  sq_dtype yt;
  int32_t* acc_out;
};
sq_status launch_bmm(const BmmArgs& a, cudaStream_t st);

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);
sq_status launch_gemm(const GemmArgs& a, cudaStream_t st);

// The GEMM in error mode (fp32 y, shapes the large-M kernel serves:
// gemm_err_ok): y is not written; each epilogue warp leaves its
// (sum (y - y_ref)^2, sum y_ref^2) in fp64 in part[2*i], part[2*i+1], and
// *nslots (at most gemm_err_max_slots()) says how many pairs were written.
bool gemm_err_ok(int64_t M, int64_t N);
int gemm_err_max_slots();
sq_status launch_gemm_err(const GemmArgs& a, const float* y_ref, double* part, int* nslots,
                          cudaStream_t st);

// sq_gemm_w8a8_noalloc: the same GEMM with its scratch in a static device
// array of kNoallocScratchBytes (gemm.cu).
constexpr size_t kNoallocScratchBytes = (size_t)8 << 20;
sq_status launch_gemm_noalloc(GemmArgs a, cudaStream_t st);

// ---------------------------------------------------------------- self test
cudaError_t launch_wait_selftest(int64_t limit_ns, cudaStream_t st);
cudaError_t launch_bounds_selftest(cudaStream_t st);

// ---------------------------------------------------------------- measurement
cudaError_t launch_mma_probe(int64_t kblocks, int grid, cudaStream_t st);
cudaError_t launch_mma_pair_probe(int64_t kblocks, int pairs, cudaStream_t st);

}  // namespace sq
