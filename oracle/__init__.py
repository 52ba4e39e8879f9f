"""CPU oracle of the smoothed W8A8 linear layer (SmoothQuant).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg (and its ``--impl reference`` arm) may import
this package.  The product path (``w8a8_int8_gemm_calib_b200``) never imports
it, and it imports nothing from the product.

The arithmetic lives in ``sq_oracle.c`` (plain single-threaded C, one fp32
rounding per operation, no contraction); this module only marshals numpy
arrays into it.  Sources are cited by tag in ``sq_oracle.h``:

* [explainer] "SmoothQuant 如何解决激活量化难题？为什么适合 W8A8？"
* [review]    "SmoothQuant：大型语言模型的精准高效训练后量化 — 深度技术评审"
* [embedded]  "嵌入式 SLM 动态权重量化：SmoothQuant 激活异常值迁移与 INT8 部署实战"

Arrays: fp32 inputs are ``np.float32``; bf16 inputs are passed as their raw
bit patterns in ``np.uint16`` and widened exactly inside the C code.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sq_oracle.c")
_HDR = os.path.join(_HERE, "sq_oracle.h")
_LIB = os.path.join(_HERE, "libsq_oracle.so")

F32 = 0
BF16 = 1
PER_TENSOR_STATIC = 0
PER_TOKEN_DYNAMIC = 1
PER_TENSOR_DYNAMIC = 2

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
          "-shared", "-fPIC", "-Wall"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (the flags above) and return the .so path."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_f = ctypes.c_float
_i = ctypes.c_int


def _declare(L):
    L.orc_delta.argtypes = [_f]
    L.orc_delta.restype = _f
    L.orc_quant.argtypes = [_f, _f]
    L.orc_quant.restype = ctypes.c_int8
    L.orc_f32_to_bf16.argtypes = [_f]
    L.orc_f32_to_bf16.restype = ctypes.c_uint16
    L.orc_layernorm_row.argtypes = [_p, _i64, _p, _p, _f, _p]
    L.orc_calib_absmax.argtypes = [_p, _i, _i64, _i64, _p, _p, _f, _p]
    L.orc_rmsnorm_row.argtypes = [_p, _i64, _p, _f, _p]
    L.orc_calib_absmax_rms.argtypes = [_p, _i, _i64, _i64, _p, _f, _p]
    L.orc_quant_act_rms.argtypes = [_p, _i, _i64, _i64, _p, _f, _i, _p, _p, _p]
    L.orc_weight_colmax.argtypes = [_p, _i, _i64, _i64, _p]
    L.orc_smooth_scales.argtypes = [_p, _p, _i64, _f, _p, _p]
    L.orc_static_delta.argtypes = [_p, _p, _i64]
    L.orc_static_delta.restype = _f
    L.orc_fuse_weights_q8.argtypes = [_p, _i, _i64, _i64, _p, _p, _p]
    L.orc_fold_ln.argtypes = [_p, _p, _p, _i64, _p, _p]
    L.orc_fold_into_producer.argtypes = [_p, _i64, _p, _p]
    L.orc_quant_act.argtypes = [_p, _i, _i64, _i64, _p, _p, _f, _p, _i, _p, _p, _p]
    L.orc_gemm_w8a8.argtypes = [_p, _p, _i64, _i64, _i64, _p, _i, _p, _p, _p, _i64,
                                _p, _p, _p]
    for fn in ("orc_layernorm_row", "orc_calib_absmax", "orc_weight_colmax",
               "orc_smooth_scales", "orc_fuse_weights_q8", "orc_fold_ln",
               "orc_quant_act", "orc_gemm_w8a8", "orc_rmsnorm_row",
               "orc_calib_absmax_rms", "orc_quant_act_rms", "orc_fold_into_producer"):
        getattr(L, fn).restype = None


def _ptr(a):
    return None if a is None else a.ctypes.data


def _typed(x):
    """(contiguous array, element-type code) for an fp32 or bf16-bits array."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"oracle inputs are float32 or bf16 bits (uint16), got {x.dtype}")


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


# ---------------------------------------------------------------- scalars

def delta(amax: float) -> float:
    """Symmetric INT8 step max(amax, 1e-7)/127 ([review] §2.2)."""
    return lib().orc_delta(amax)


def quant(v: float, d: float) -> int:
    """Q(v; d): v * (1/d), round half to even, clamp [-127, 127]."""
    return lib().orc_quant(v, d)


def f32_to_bf16_bits(x) -> np.ndarray:
    """Round fp32 values to bf16 (nearest even); returns the uint16 patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    L = lib()
    out = np.empty(x.shape, dtype=np.uint16)
    flat, of = x.reshape(-1), out.reshape(-1)
    for i in range(flat.size):
        of[i] = L.orc_f32_to_bf16(float(flat[i]))
    return out


# ---------------------------------------------------------------- steps

def layernorm_row(x, g, b, eps=1e-5):
    x, g, b = _f32(x), _f32(g), _f32(b)
    y = np.empty_like(x)
    lib().orc_layernorm_row(_ptr(x), x.size, _ptr(g), _ptr(b), eps, _ptr(y))
    return y


def rmsnorm_row(x, g, eps=1e-5):
    x, g = _f32(x), _f32(g)
    y = np.empty_like(x)
    lib().orc_rmsnorm_row(_ptr(x), x.size, _ptr(g), eps, _ptr(y))
    return y


def calib_absmax_rms(x, gamma, eps=1e-5, amax=None):
    """S1 through an RMSNorm with the original gamma."""
    x, xt = _typed(x)
    T, K = x.shape
    amax = np.zeros(K, np.float32) if amax is None else np.array(amax, np.float32)
    gamma = _f32(gamma)
    lib().orc_calib_absmax_rms(_ptr(x), xt, T, K, _ptr(gamma), eps, _ptr(amax))
    return amax


def quant_act_rms(x, gamma_s, eps=1e-5, per_token=True, static_delta=None,
                  per_tensor_dynamic=False):
    """S5 with y = RMSNorm(x; gamma_s): (xq, act_scale, n_clipped)."""
    x, xt = _typed(x)
    T, K = x.shape
    gamma_s = _f32(gamma_s)
    if per_tensor_dynamic:
        act, gran = np.zeros(1, np.float32), PER_TENSOR_DYNAMIC
    elif per_token:
        act, gran = np.empty(T, np.float32), PER_TOKEN_DYNAMIC
    else:
        act, gran = np.array([static_delta], np.float32), PER_TENSOR_STATIC
    xq = np.empty((T, K), np.int8)
    ncl = ctypes.c_int64(0)
    lib().orc_quant_act_rms(_ptr(x), xt, T, K, _ptr(gamma_s), eps, gran, _ptr(act),
                            _ptr(xq), ctypes.addressof(ncl))
    return xq, act, int(ncl.value)


def calib_absmax(x, gamma=None, beta=None, eps=1e-5, amax=None):
    """S1: running per-input-channel absmax of X (or of LN(X)) over tokens."""
    x, xt = _typed(x)
    T, K = x.shape
    amax = np.zeros(K, np.float32) if amax is None else np.array(amax, np.float32)
    gamma, beta = _f32(gamma), _f32(beta)
    lib().orc_calib_absmax(_ptr(x), xt, T, K, _ptr(gamma), _ptr(beta), eps, _ptr(amax))
    return amax


def weight_colmax(w):
    w, wt = _typed(w)
    N, K = w.shape
    out = np.empty(K, np.float32)
    lib().orc_weight_colmax(_ptr(w), wt, N, K, _ptr(out))
    return out


def smooth_scales(amax_x, amax_w, alpha):
    """S2: eq. (4) -> (s, inv_s), fp32."""
    amax_x, amax_w = _f32(amax_x), _f32(amax_w)
    K = amax_x.size
    s = np.empty(K, np.float32)
    inv_s = np.empty(K, np.float32)
    lib().orc_smooth_scales(_ptr(amax_x), _ptr(amax_w), K, float(alpha), _ptr(s), _ptr(inv_s))
    return s, inv_s


def static_delta(amax_x, s):
    """S3: static per-tensor activation step from calibration peaks."""
    amax_x, s = _f32(amax_x), _f32(s)
    return np.float32(lib().orc_static_delta(_ptr(amax_x), _ptr(s), amax_x.size))


def fuse_weights_q8(w, s):
    """S4: W_hat = W*s, per-output-channel INT8 -> (wq int8 [N,K], w_scale [N])."""
    w, wt = _typed(w)
    N, K = w.shape
    s = _f32(s)
    wq = np.empty((N, K), np.int8)
    ws = np.empty(N, np.float32)
    lib().orc_fuse_weights_q8(_ptr(w), wt, N, K, _ptr(s), _ptr(wq), _ptr(ws))
    return wq, ws


def bmm_w8a8(xq, wq, act_scale, w_scale, per_token=True, w_per_channel=True, out_bf16=False):
    """S6 applied to each batch b of xq [B, M, K] and wq [B, N, K]: act_scale
    [B*M] (per token) or [B]; w_scale [B*N] (per channel) or [B].  Returns
    (y [B, M, N], acc [B, M, N])."""
    xq = np.ascontiguousarray(xq, np.int8)
    wq = np.ascontiguousarray(wq, np.int8)
    B, M, _ = xq.shape
    N = wq.shape[1]
    act_scale, w_scale = _f32(act_scale), _f32(w_scale)
    ys, accs = [], []
    for b in range(B):
        a = act_scale[b * M:(b + 1) * M] if per_token else act_scale[b:b + 1]
        w = w_scale[b * N:(b + 1) * N] if w_per_channel else np.full(N, w_scale[b], np.float32)
        y, acc = gemm_w8a8(xq[b], wq[b], a, w, per_token=per_token, out_bf16=out_bf16)
        ys.append(y)
        accs.append(acc)
    return np.stack(ys), np.stack(accs)


def fold_into_producer(s, w_scale, bias=None):
    """The producer's per-output-channel scale (and bias) divided by s."""
    s = _f32(s)
    ws = np.array(w_scale, np.float32)
    b = None if bias is None else np.array(bias, np.float32)
    lib().orc_fold_into_producer(_ptr(s), s.size, _ptr(ws), _ptr(b))
    return ws, b


def fold_ln(gamma, beta, s):
    """S4: gamma/s, beta/s ([embedded] §二)."""
    gamma, beta, s = _f32(gamma), _f32(beta), _f32(s)
    K = s.size
    g2 = np.empty(K, np.float32) if gamma is not None else None
    b2 = np.empty(K, np.float32) if beta is not None else None
    lib().orc_fold_ln(_ptr(gamma), _ptr(beta), _ptr(s), K, _ptr(g2), _ptr(b2))
    return g2, b2


def quant_act(x, gamma_s=None, beta_s=None, eps=1e-5, inv_s=None,
              per_token=True, static_delta=None, per_tensor_dynamic=False):
    """S5: returns (xq int8 [T,K], act_scale [T] or [1], n_clipped).
    per_tensor_dynamic: one step from the peak of the whole call (O2)."""
    x, xt = _typed(x)
    T, K = x.shape
    gamma_s, beta_s, inv_s = _f32(gamma_s), _f32(beta_s), _f32(inv_s)
    if per_tensor_dynamic:
        act = np.zeros(1, np.float32)
        gran = PER_TENSOR_DYNAMIC
    elif per_token:
        act = np.empty(T, np.float32)
        gran = PER_TOKEN_DYNAMIC
    else:
        act = np.array([static_delta], np.float32)
        gran = PER_TENSOR_STATIC
    xq = np.empty((T, K), np.int8)
    ncl = ctypes.c_int64(0)
    lib().orc_quant_act(_ptr(x), xt, T, K, _ptr(gamma_s), _ptr(beta_s), eps,
                        _ptr(inv_s), gran, _ptr(act), _ptr(xq), ctypes.addressof(ncl))
    return xq, act, int(ncl.value)


def gemm_w8a8(xq, wq, act_scale, w_scale, per_token=True, rows=None,
              out_bf16=False, bias=None):
    """S6: returns (y, acc): y fp32 or bf16 bits (uint16), acc int32.

    rows: optional token indices; only those rows are computed (in order).
    bias: optional [N] fp32 added after the dequantization.
    """
    xq = np.ascontiguousarray(xq, np.int8)
    wq = np.ascontiguousarray(wq, np.int8)
    M, K = xq.shape
    N = wq.shape[0]
    act_scale, w_scale, bias = _f32(act_scale), _f32(w_scale), _f32(bias)
    r = None if rows is None else np.ascontiguousarray(rows, np.int64)
    R = M if r is None else r.size
    acc = np.empty((R, N), np.int32)
    yf = None if out_bf16 else np.empty((R, N), np.float32)
    yb = np.empty((R, N), np.uint16) if out_bf16 else None
    lib().orc_gemm_w8a8(_ptr(xq), _ptr(wq), M, N, K, _ptr(act_scale), int(per_token),
                        _ptr(w_scale), _ptr(bias), _ptr(r), R, _ptr(yf), _ptr(yb), _ptr(acc))
    return (yb if out_bf16 else yf), acc


def output_error(y, y_ref):
    """Relative Frobenius error ||y - y_ref|| / ||y_ref||, sums in fp64 (the
    layer-output error that alpha is chosen by)."""
    y = np.asarray(y, np.float64)
    r = np.asarray(y_ref, np.float64)
    num = float(np.sum((y - r) ** 2))
    den = float(np.sum(r * r))
    if den > 0:
        return math.sqrt(num / den)
    return math.inf if num > 0 else 0.0


def alpha_error(amax_x, w, x, y_ref, alpha, gamma=None, beta=None, eps=1e-5,
                gran="token"):
    """The smoothed W8A8 layer at one alpha, built from the calibration peaks
    amax_x: eq. (4), the fold, the quantizer at granularity gran ("token",
    "static", "tensor"), the GEMM in fp32; returns its output_error against
    y_ref."""
    s, inv_s = smooth_scales(amax_x, weight_colmax(w), alpha)
    wq, ws = fuse_weights_q8(w, s)
    kw = dict(per_token=gran == "token", per_tensor_dynamic=gran == "tensor",
              static_delta=static_delta(amax_x, s) if gran == "static" else None)
    if gamma is not None:
        g2, b2 = fold_ln(gamma, beta, s)
        xq, act, _ = quant_act(x, g2, b2, eps, **kw)
    else:
        xq, act, _ = quant_act(x, inv_s=inv_s, **kw)
    y, _ = gemm_w8a8(xq, wq, act, ws, per_token=gran == "token")
    return output_error(y, y_ref)
