"""ctypes binding of libsq_b200.so (the C ABI in include/sq.h).

Argument marshalling only: every function takes torch tensors that already
live on the GPU, passes their data pointers and the current CUDA stream to
the C entry point of the same name, and raises SQError on a non-OK status.
No step of the computation runs here, and there is no CPU fallback: if the
compiled library is missing, importing this module fails.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# SQ_B200_LIB may name another build of the same library, such as the
# bounds-checked libsq_b200_debug.so (build.py --debug-bounds)
LIB_PATH = os.environ.get("SQ_B200_LIB") or os.path.join(_HERE, "libsq_b200.so")

SQ_OK = 0
SQ_ERR_INVALID_ARG = 1
SQ_ERR_SHAPE = 2
SQ_ERR_ALIGN = 3
SQ_ERR_DTYPE = 4
SQ_ERR_UNSUPPORTED = 5
SQ_ERR_CUDA = 6
SQ_ERR_TIMEOUT = 7
SQ_ERR_WORKSPACE = 8
SQ_ERR_BOUNDS = 9

SQ_F32 = 0
SQ_BF16 = 1
SQ_ACT_PER_TENSOR_STATIC = 0
SQ_ACT_PER_TOKEN_DYNAMIC = 1
SQ_ACT_PER_TENSOR_DYNAMIC = 2

EXPORTS = [
    "sq_calib_absmax", "sq_smooth_scales", "sq_fuse_weights_q8",
    "sq_ln_smooth_quant_act", "sq_gemm_workspace_bytes", "sq_gemm_w8a8",
    "sq_sync_status", "sq_status_string", "sq_last_error",
    "sq_selftest_bounded_wait", "sq_gemm_w8a8_noalloc", "sq_gemm_w8a8_bias",
    "sq_calib_absmax_rms", "sq_rms_smooth_quant_act", "sq_fold_into_producer",
    "sq_alpha_sweep_workspace_bytes", "sq_alpha_sweep", "sq_bmm_w8a8",
    "sq_weight_colmax", "sq_smooth_scales_peaks", "sq_probe_mma_i8", "sq_probe_mma_i8_pair",
    "sq_debug_bounds_enabled", "sq_selftest_bounds_check",
]


class SQError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}: {detail}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python w8a8_int8_gemm_calib_b200/build.py` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    p, i64, f, i, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int, ctypes.c_size_t
    st = ctypes.c_int
    L.sq_calib_absmax.argtypes = [p, i, i64, i64, p, p, f, p, p]
    L.sq_calib_absmax_rms.argtypes = [p, i, i64, i64, p, f, p, p]
    L.sq_fold_into_producer.argtypes = [p, i64, p, p, p]
    L.sq_weight_colmax.argtypes = [p, i, i64, i64, p, p]
    L.sq_smooth_scales_peaks.argtypes = [p, p, i64, f, p, p, p, p]
    L.sq_bmm_w8a8.argtypes = [p, p, i64, i64, i64, i64, p, i, p, i, p, i, p, p]
    L.sq_alpha_sweep_workspace_bytes.argtypes = [i64, i64, i64]
    L.sq_alpha_sweep_workspace_bytes.restype = sz
    L.sq_alpha_sweep.argtypes = [p, p, i, i64, i64, p, i, i64, p, p, f, p, p, i, i, p, p, sz, p]
    L.sq_rms_smooth_quant_act.argtypes = [p, i, i64, i64, p, f, i, p, p, p, p]
    L.sq_smooth_scales.argtypes = [p, p, i, i64, i64, f, p, p, p, p]
    L.sq_fuse_weights_q8.argtypes = [p, i, i64, i64, p, p, p, p, p, p, p, p]
    L.sq_ln_smooth_quant_act.argtypes = [p, i, i64, i64, p, p, f, p, i, p, p, p, p]
    L.sq_gemm_workspace_bytes.argtypes = [i64, i64, i64]
    L.sq_gemm_workspace_bytes.restype = sz
    L.sq_gemm_w8a8.argtypes = [p, p, i64, i64, i64, p, i, p, p, i, p, p, sz, p]
    L.sq_gemm_w8a8_bias.argtypes = [p, p, i64, i64, i64, p, i, p, p, p, i, p, p, sz, p]
    L.sq_sync_status.argtypes = [p]
    L.sq_status_string.argtypes = [st]
    L.sq_status_string.restype = ctypes.c_char_p
    L.sq_last_error.argtypes = []
    L.sq_last_error.restype = ctypes.c_char_p
    L.sq_selftest_bounded_wait.argtypes = [i64, p]
    L.sq_probe_mma_i8.argtypes = [i64, i, p]
    L.sq_probe_mma_i8_pair.argtypes = [i64, i, p]
    L.sq_debug_bounds_enabled.argtypes = []
    L.sq_debug_bounds_enabled.restype = i
    L.sq_selftest_bounds_check.argtypes = [p]
    L.sq_gemm_w8a8_noalloc.argtypes = [p, p, i64, i64, i64, p, i, p, p, i, p, p]
    for fn in ("sq_calib_absmax", "sq_smooth_scales", "sq_fuse_weights_q8",
               "sq_ln_smooth_quant_act", "sq_gemm_w8a8", "sq_sync_status",
               "sq_selftest_bounded_wait", "sq_gemm_w8a8_noalloc", "sq_gemm_w8a8_bias",
               "sq_calib_absmax_rms", "sq_rms_smooth_quant_act", "sq_fold_into_producer",
               "sq_alpha_sweep", "sq_bmm_w8a8", "sq_weight_colmax", "sq_smooth_scales_peaks",
               "sq_probe_mma_i8", "sq_probe_mma_i8_pair", "sq_selftest_bounds_check"):
        getattr(L, fn).restype = st
    return L


lib = _load()


def status_string(s: int) -> str:
    return lib.sq_status_string(s).decode()


def last_error() -> str:
    return lib.sq_last_error().decode()


def check(s: int, where: str) -> None:
    if s != SQ_OK:
        raise SQError(s, where, last_error())
