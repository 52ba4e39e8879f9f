"""B200 (sm_100a) smoothed W8A8 linear layer: the SmoothQuant hot path.

Thin torch-facing wrappers over the C ABI of include/sq.h, one per entry
point and with the same names.  They only marshal arguments (data pointers,
sizes, the current CUDA stream); every step of the computation runs in the
library's CUDA kernels.  Tensors must be contiguous CUDA tensors, 16-byte
aligned (fresh torch allocations are).

Sources:
* "SmoothQuant 如何解决激活量化难题？为什么适合 W8A8？" §三, §四
* "SmoothQuant：大型语言模型的精准高效训练后量化 — 深度技术评审" §2.2, §2.5, §2.6,
  §5.1 eq. (3), §5.3 eq. (4), §5.5, §6.3
* "嵌入式 SLM 动态权重量化：SmoothQuant 激活异常值迁移与 INT8 部署实战" §二, §三
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import (SQ_ACT_PER_TENSOR_DYNAMIC, SQ_ACT_PER_TENSOR_STATIC, SQ_ACT_PER_TOKEN_DYNAMIC, SQ_BF16,
                   SQ_F32, SQError, check, lib)

__all__ = [
    "sq_calib_absmax", "sq_smooth_scales", "sq_fuse_weights_q8",
    "sq_ln_smooth_quant_act", "sq_gemm_workspace_bytes", "sq_gemm_w8a8",
    "sq_sync_status", "sq_selftest_bounded_wait", "SQError", "Workspace",
    "sq_calib_absmax_rms", "sq_rms_smooth_quant_act", "sq_fold_into_producer",
    "sq_alpha_sweep_workspace_bytes", "sq_alpha_sweep", "sq_bmm_w8a8",
    "sq_weight_colmax", "sq_smooth_scales_peaks", "sq_probe_mma_i8", "sq_probe_mma_i8_pair",
    "sq_debug_bounds_enabled", "sq_selftest_bounds_check",
]


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SQ_F32
    if t.dtype == torch.bfloat16:
        return SQ_BF16
    raise TypeError(f"expected float32 or bfloat16, got {t.dtype}")


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def sq_calib_absmax(x, amax, ln_gamma=None, ln_beta=None, ln_eps=1e-5, stream=None):
    """Running per-input-channel peak of X (or of LN(X)) over tokens; amax [K] fp32 in/out."""
    T, K = x.shape
    check(lib.sq_calib_absmax(_ptr(x), _dt(x), T, K, _ptr(ln_gamma), _ptr(ln_beta),
                              ln_eps, _ptr(amax), _stream(stream)), "sq_calib_absmax")
    return amax


def sq_calib_absmax_rms(x, amax, gamma, eps=1e-5, stream=None):
    """Running per-input-channel peak of RMSNorm(X; gamma) over tokens."""
    T, K = x.shape
    check(lib.sq_calib_absmax_rms(_ptr(x), _dt(x), T, K, _ptr(gamma), eps, _ptr(amax),
                                  _stream(stream)), "sq_calib_absmax_rms")
    return amax


def sq_smooth_scales(amax_x, w, alpha, s, inv_s, act_delta_static=None, stream=None):
    """eq. (4) smoothing factors s, 1/s (and the static activation step)."""
    N, K = w.shape
    check(lib.sq_smooth_scales(_ptr(amax_x), _ptr(w), _dt(w), N, K, float(alpha), _ptr(s),
                               _ptr(inv_s), _ptr(act_delta_static), _stream(stream)),
          "sq_smooth_scales")
    return s, inv_s


def sq_weight_colmax(w, amax_w, stream=None):
    """amax_w[k] = max_n |W[n,k]| (the weight half of eq. (4)'s peaks)."""
    N, K = w.shape
    check(lib.sq_weight_colmax(_ptr(w), _dt(w), N, K, _ptr(amax_w), _stream(stream)),
          "sq_weight_colmax")
    return amax_w


def sq_smooth_scales_peaks(amax_x, amax_w, alpha, s, inv_s, act_delta_static=None, stream=None):
    """eq. (4) from both sets of peaks: s, 1/s (and the static step)."""
    K = amax_x.numel()
    check(lib.sq_smooth_scales_peaks(_ptr(amax_x), _ptr(amax_w), K, float(alpha), _ptr(s),
                                     _ptr(inv_s), _ptr(act_delta_static), _stream(stream)),
          "sq_smooth_scales_peaks")
    return s, inv_s


def sq_fuse_weights_q8(w, s, wq, w_scale, gamma=None, beta=None, gamma_out=None,
                       beta_out=None, stream=None):
    """W*s -> per-output-channel INT8 (wq, w_scale); gamma/s, beta/s."""
    N, K = w.shape
    check(lib.sq_fuse_weights_q8(_ptr(w), _dt(w), N, K, _ptr(s), _ptr(wq), _ptr(w_scale),
                                 _ptr(gamma), _ptr(beta), _ptr(gamma_out), _ptr(beta_out),
                                 _stream(stream)), "sq_fuse_weights_q8")
    return wq, w_scale


def sq_ln_smooth_quant_act(x, xq, act_scale, gamma_s=None, beta_s=None, ln_eps=1e-5,
                           inv_s=None, per_token=True, n_clipped=None, stream=None,
                           per_tensor_dynamic=False):
    """Fused LN + smoothing + symmetric INT8 quantizer -> xq (and act_scale).
    per_token: one step per token; else the step in act_scale[0] (static), or
    with per_tensor_dynamic one step from the peak of the whole call."""
    T, K = x.shape
    if per_tensor_dynamic:
        gran = SQ_ACT_PER_TENSOR_DYNAMIC
    else:
        gran = SQ_ACT_PER_TOKEN_DYNAMIC if per_token else SQ_ACT_PER_TENSOR_STATIC
    check(lib.sq_ln_smooth_quant_act(_ptr(x), _dt(x), T, K, _ptr(gamma_s), _ptr(beta_s),
                                     ln_eps, _ptr(inv_s), gran, _ptr(act_scale), _ptr(xq),
                                     _ptr(n_clipped), _stream(stream)),
          "sq_ln_smooth_quant_act")
    return xq, act_scale


def sq_rms_smooth_quant_act(x, xq, act_scale, gamma_s, eps=1e-5, per_token=True,
                            n_clipped=None, stream=None, per_tensor_dynamic=False):
    """RMSNorm (gamma_s = gamma / s) + symmetric INT8 quantizer -> xq (and
    act_scale), granularities as sq_ln_smooth_quant_act."""
    T, K = x.shape
    if per_tensor_dynamic:
        gran = SQ_ACT_PER_TENSOR_DYNAMIC
    else:
        gran = SQ_ACT_PER_TOKEN_DYNAMIC if per_token else SQ_ACT_PER_TENSOR_STATIC
    check(lib.sq_rms_smooth_quant_act(_ptr(x), _dt(x), T, K, _ptr(gamma_s), eps, gran,
                                      _ptr(act_scale), _ptr(xq), _ptr(n_clipped),
                                      _stream(stream)), "sq_rms_smooth_quant_act")
    return xq, act_scale


def sq_fold_into_producer(s, w_scale, bias=None, stream=None):
    """1/s folded into the producing linear: w_scale /= s, bias /= s (in place)."""
    K = s.numel()
    check(lib.sq_fold_into_producer(_ptr(s), K, _ptr(w_scale), _ptr(bias), _stream(stream)),
          "sq_fold_into_producer")
    return w_scale, bias


def sq_alpha_sweep_workspace_bytes(M, N, K) -> int:
    return int(lib.sq_alpha_sweep_workspace_bytes(M, N, K))


def sq_alpha_sweep(amax_x, w, x, y_ref, alphas, ln_gamma=None, ln_beta=None, ln_eps=1e-5,
                   per_token=True, per_tensor_dynamic=False, workspace=None, stream=None):
    """Layer-output error of the smoothed W8A8 layer at each alpha: a CUDA
    tensor of len(alphas) doubles, ||y - y_ref|| / ||y_ref||."""
    N, K = w.shape
    M = x.shape[0]
    if per_tensor_dynamic:
        gran = SQ_ACT_PER_TENSOR_DYNAMIC
    else:
        gran = SQ_ACT_PER_TOKEN_DYNAMIC if per_token else SQ_ACT_PER_TENSOR_STATIC
    need = sq_alpha_sweep_workspace_bytes(M, N, K)
    ws = workspace.get(need) if isinstance(workspace, Workspace) else workspace
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=x.device)
    a = (ctypes.c_float * len(alphas))(*[float(v) for v in alphas])
    err = torch.empty(len(alphas), dtype=torch.float64, device=x.device)
    check(lib.sq_alpha_sweep(_ptr(amax_x), _ptr(w), _dt(w), N, K, _ptr(x), _dt(x), M,
                             _ptr(ln_gamma), _ptr(ln_beta), ln_eps, _ptr(y_ref), a, len(alphas),
                             gran, _ptr(err), _ptr(ws), ws.numel() * ws.element_size(),
                             _stream(stream)), "sq_alpha_sweep")
    return err


def sq_bmm_w8a8(xq, wq, act_scale, w_scale, y, per_token=True, w_per_channel=True,
                acc_out=None, stream=None):
    """Batched INT8 GEMM: y[b] = (float)(xq[b] @ wq[b]^T) * (as * ws), xq
    [batch, M, K], wq [batch, N, K], y [batch, M, N]."""
    B, M, K = xq.shape
    N = wq.shape[1]
    check(lib.sq_bmm_w8a8(_ptr(xq), _ptr(wq), B, M, N, K, _ptr(act_scale), int(per_token),
                          _ptr(w_scale), int(w_per_channel), _ptr(y), _dt(y), _ptr(acc_out),
                          _stream(stream)), "sq_bmm_w8a8")
    return y


def sq_gemm_workspace_bytes(M, N, K) -> int:
    return int(lib.sq_gemm_workspace_bytes(M, N, K))


class Workspace:
    """Device scratch for sq_gemm_w8a8, grown on demand.  The GEMM needs no
    particular contents: each call resets the part it counts with."""

    def __init__(self, device=None):
        self.device = device
        self.buf = None

    def get(self, nbytes: int):
        if nbytes == 0:
            return None
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(nbytes, dtype=torch.uint8, device=self.device or "cuda")
        return self.buf


def sq_gemm_w8a8(xq, wq, act_scale, w_scale, y, per_token=True, acc_out=None,
                 workspace=None, stream=None, bias=None):
    """y = (float)(xq @ wq^T) * (act_scale[t] * w_scale[n]) (+ bias[n]);
    y fp32 or bf16.  With a bias this calls sq_gemm_w8a8_bias."""
    M, K = xq.shape
    N = wq.shape[0]
    need = sq_gemm_workspace_bytes(M, N, K)
    ws = None
    if need:
        if workspace is None:
            raise ValueError(f"sq_gemm_w8a8 needs a workspace of {need} bytes")
        ws = workspace.get(need) if isinstance(workspace, Workspace) else workspace
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    if bias is None:
        check(lib.sq_gemm_w8a8(_ptr(xq), _ptr(wq), M, N, K, _ptr(act_scale), int(per_token),
                               _ptr(w_scale), _ptr(y), _dt(y), _ptr(acc_out), _ptr(ws),
                               nbytes, _stream(stream)), "sq_gemm_w8a8")
    else:
        check(lib.sq_gemm_w8a8_bias(_ptr(xq), _ptr(wq), M, N, K, _ptr(act_scale),
                                    int(per_token), _ptr(w_scale), _ptr(bias), _ptr(y), _dt(y),
                                    _ptr(acc_out), _ptr(ws), nbytes, _stream(stream)),
              "sq_gemm_w8a8_bias")
    return y


def sq_sync_status(stream=None):
    """Synchronize the stream and raise SQError if a kernel recorded a fault."""
    check(lib.sq_sync_status(_stream(stream)), "sq_sync_status")


def sq_selftest_bounded_wait(limit_ns: int, stream=None):
    check(lib.sq_selftest_bounded_wait(int(limit_ns), _stream(stream)),
          "sq_selftest_bounded_wait")


def sq_probe_mma_i8(kblocks: int, grid: int, stream=None):
    """Launch the INT8 tensor-core rate probe: grid CTAs, each issuing
    kblocks x 4 tcgen05.mma kind::i8 steps of 128 x 256 x 32 (8,388,608 ops
    per k-block).  Returns the op count; the caller times the launch."""
    check(lib.sq_probe_mma_i8(int(kblocks), int(grid), _stream(stream)), "sq_probe_mma_i8")
    return 8388608 * int(kblocks) * int(grid)


def sq_probe_mma_i8_pair(kblocks: int, pairs: int, stream=None):
    """Launch the CTA-pair INT8 tensor-core rate probe: `pairs` clusters of two
    CTAs issuing kblocks x 4 tcgen05.mma.cta_group::2 steps of 256 x 256 x 32
    (16,777,216 ops per k-block per pair).  Returns the op count."""
    check(lib.sq_probe_mma_i8_pair(int(kblocks), int(pairs), _stream(stream)),
          "sq_probe_mma_i8_pair")
    return 16777216 * int(kblocks) * int(pairs)


def sq_debug_bounds_enabled() -> bool:
    """True for the bounds-checked build (libsq_b200_debug.so)."""
    return bool(lib.sq_debug_bounds_enabled())


def sq_selftest_bounds_check(stream=None):
    """Launch the bounds-check self-test (one thread checks an offset at
    its tensor's end, touching no memory); sq_sync_status() then raises
    SQ_ERR_BOUNDS in the bounds-checked build and nothing otherwise."""
    check(lib.sq_selftest_bounds_check(_stream(stream)), "sq_selftest_bounds_check")
