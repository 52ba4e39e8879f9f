"""Host-side checks of the C ABI: the library loads, exports every entry point
include/sq.h declares, and rejects bad arguments before anything reaches the
GPU (no device is needed: every call here fails or is empty before the
first CUDA call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from w8a8_int8_gemm_calib_b200 import _lib

    return _lib


def declared_functions():
    src = open(os.path.join(ROOT, "include", "sq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sq_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "sq_gemm_w8a8" in names and len(names) >= 10
    raw = ctypes.CDLL(lib.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), f"{n} declared in include/sq.h but not exported"
    assert set(names) == set(lib.EXPORTS)


def test_status_strings(lib):
    for code in range(10):
        assert lib.status_string(code).startswith("SQ_")
    assert lib.status_string(42) == "SQ_ERR_UNKNOWN"


# fake, never dereferenced device addresses
A = 1 << 20
A2 = (1 << 20) + 4096
MIS = (1 << 20) + 8


def test_calib_absmax_checks(lib):
    L = lib.lib
    assert L.sq_calib_absmax(A, 1, 10, 17, None, None, 1e-5, A2, None) == lib.SQ_ERR_SHAPE
    assert L.sq_calib_absmax(A, 1, 10, 0, None, None, 1e-5, A2, None) == lib.SQ_ERR_SHAPE
    assert L.sq_calib_absmax(A, 1, 10, 133152, None, None, 1e-5, A2, None) == lib.SQ_ERR_SHAPE
    assert L.sq_calib_absmax(A, 1, -1, 16, None, None, 1e-5, A2, None) == lib.SQ_ERR_SHAPE
    assert L.sq_calib_absmax(A, 7, 10, 16, None, None, 1e-5, A2, None) == lib.SQ_ERR_DTYPE
    assert L.sq_calib_absmax(None, 1, 10, 16, None, None, 1e-5, A2, None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_calib_absmax(MIS, 1, 10, 16, None, None, 1e-5, A2, None) == lib.SQ_ERR_ALIGN
    assert L.sq_calib_absmax(A, 1, 10, 16, None, A2, 1e-5, A2, None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_calib_absmax(A, 1, 10, 16, A2, None, -1.0, A2, None) == lib.SQ_ERR_INVALID_ARG
    assert "multiple of 16" in (L.sq_calib_absmax(A, 1, 1, 24, None, None, 0, A2, None)
                                and lib.last_error())
    # empty problem: nothing to do, nothing launched
    assert L.sq_calib_absmax(A, 1, 0, 16, None, None, 1e-5, A2, None) == lib.SQ_OK


def test_smooth_scales_checks(lib):
    L = lib.lib
    for bad_alpha in (-0.1, 1.5, float("nan")):
        assert L.sq_smooth_scales(A, A, 1, 4, 16, bad_alpha, A2, A2, None, None) == \
            lib.SQ_ERR_INVALID_ARG
    assert L.sq_smooth_scales(A, A, 1, 4, 20, 0.5, A2, A2, None, None) == lib.SQ_ERR_SHAPE
    assert L.sq_smooth_scales(A, A, 1, 4, 16, 0.5, None, A2, None, None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_smooth_scales(A, A, 1, 4, 16, 0.5, A2, A2, MIS, None) == lib.SQ_ERR_ALIGN


def test_fuse_weights_checks(lib):
    L = lib.lib
    assert L.sq_fuse_weights_q8(A, 1, 4, 16, None, A2, A2, None, None, None, None, None) == \
        lib.SQ_ERR_INVALID_ARG
    assert L.sq_fuse_weights_q8(A, 1, 4, 16, A, None, A2, None, None, None, None, None) == \
        lib.SQ_ERR_INVALID_ARG
    assert L.sq_fuse_weights_q8(A, 1, -4, 16, A, A2, A2, None, None, None, None, None) == \
        lib.SQ_ERR_SHAPE
    assert L.sq_fuse_weights_q8(A, 1, 4, 16, A, A2, A2, MIS, None, None, None, None) == \
        lib.SQ_ERR_ALIGN


def test_quant_act_checks(lib):
    L = lib.lib
    assert L.sq_ln_smooth_quant_act(A, 1, 4, 16, None, None, 1e-5, None, 9, A2, A2, None,
                                    None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_ln_smooth_quant_act(A, 1, 4, 16, A, None, 1e-5, A2, 1, A2, A2, None,
                                    None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_ln_smooth_quant_act(A, 1, 4, 16, None, None, 1e-5, None, 1, A2, A2, A + 4,
                                    None) == lib.SQ_ERR_ALIGN
    assert L.sq_ln_smooth_quant_act(A, 1, 4, 40, None, None, 1e-5, None, 1, A2, A2, None,
                                    None) == lib.SQ_ERR_SHAPE
    assert L.sq_ln_smooth_quant_act(A, 1, 0, 16, None, None, 1e-5, None, 1, A2, A2, None,
                                    None) == lib.SQ_OK
    # per-tensor dynamic (2) is a granularity; 3 is not; its checks are the same
    assert L.sq_ln_smooth_quant_act(A, 1, 4, 16, None, None, 1e-5, None, 3, A2, A2, None,
                                    None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_ln_smooth_quant_act(A, 1, 4, 16, None, None, 1e-5, None, 2, MIS, A2, None,
                                    None) == lib.SQ_ERR_ALIGN
    assert L.sq_ln_smooth_quant_act(A, 1, 0, 16, None, None, 1e-5, None, 2, A2, A2, None,
                                    None) == lib.SQ_OK
    assert lib.SQ_ACT_PER_TENSOR_DYNAMIC == 2


def test_rmsnorm_checks(lib):
    L = lib.lib
    # gamma is required; eps finite and >= 0; the rest as the LayerNorm calls
    assert L.sq_calib_absmax_rms(A, 1, 4, 16, None, 1e-5, A2, None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_calib_absmax_rms(A, 1, 4, 16, A2, -1.0, A2, None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_calib_absmax_rms(A, 1, 4, 24, A2, 1e-5, A2, None) == lib.SQ_ERR_SHAPE
    assert L.sq_calib_absmax_rms(A, 1, 0, 16, A2, 1e-5, A2, None) == lib.SQ_OK
    assert L.sq_rms_smooth_quant_act(A, 1, 4, 16, None, 1e-5, 1, A2, A2, None, None) == \
        lib.SQ_ERR_INVALID_ARG
    assert "sq_rms_smooth_quant_act" in lib.last_error()
    assert L.sq_rms_smooth_quant_act(A, 1, 4, 16, A2, 1e-5, 7, A2, A2, None, None) == \
        lib.SQ_ERR_INVALID_ARG
    assert L.sq_rms_smooth_quant_act(A, 1, 4, 16, MIS, 1e-5, 1, A2, A2, None, None) == \
        lib.SQ_ERR_ALIGN
    assert L.sq_rms_smooth_quant_act(A, 1, 0, 16, A2, 1e-5, 2, A2, A2, None, None) == lib.SQ_OK


def test_fold_into_producer_checks(lib):
    L = lib.lib
    assert L.sq_fold_into_producer(None, 16, A2, None, None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_fold_into_producer(A, 16, None, None, None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_fold_into_producer(A, 16, A2, MIS, None) == lib.SQ_ERR_ALIGN
    assert L.sq_fold_into_producer(A, -1, A2, None, None) == lib.SQ_ERR_SHAPE
    assert L.sq_fold_into_producer(A, 0, A2, None, None) == lib.SQ_OK


def test_alpha_sweep_checks(lib):
    import ctypes as C

    L = lib.lib
    need = L.sq_alpha_sweep_workspace_bytes(64, 256, 1024)
    assert need > 256 * 1024 + 64 * 1024 + 4 * 64 * 256
    assert L.sq_alpha_sweep_workspace_bytes(0, 256, 1024) == 0
    good = (C.c_float * 2)(0.0, 0.5)
    bad = (C.c_float * 2)(0.5, 1.5)
    args = lambda al, n, gran, ws_bytes: (A, A, 1, 256, 1024, A, 1, 64, None, None, 1e-5, A,
                                          al, n, gran, A2, A2, ws_bytes, None)
    assert L.sq_alpha_sweep(*args(bad, 2, 1, need)) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_alpha_sweep(*args(good, 2, 5, need)) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_alpha_sweep(*args(good, 2, 1, need - 1)) == lib.SQ_ERR_WORKSPACE
    assert L.sq_alpha_sweep(*args(good, 0, 1, need)) == lib.SQ_OK


def test_bmm_checks(lib):
    L = lib.lib
    assert L.sq_bmm_w8a8(A, A, 2, 4, 4, 24, A2, 1, A2, 1, A2, 1, None, None) == lib.SQ_ERR_SHAPE
    assert L.sq_bmm_w8a8(A, A, -1, 4, 4, 16, A2, 1, A2, 1, A2, 1, None, None) == lib.SQ_ERR_SHAPE
    assert L.sq_bmm_w8a8(A, None, 2, 4, 4, 16, A2, 1, A2, 1, A2, 1, None, None) == \
        lib.SQ_ERR_INVALID_ARG
    assert L.sq_bmm_w8a8(A, A, 2, 4, 4, 16, A2, 1, A2, 1, MIS, 1, None, None) == lib.SQ_ERR_ALIGN
    assert L.sq_bmm_w8a8(A, A, 2, 4, 4, 16, A2, 1, A2, 1, A2, 9, None, None) == lib.SQ_ERR_DTYPE
    assert L.sq_bmm_w8a8(A, A, 0, 4, 4, 16, A2, 1, A2, 1, A2, 1, None, None) == lib.SQ_OK


def test_weight_peaks_and_scales_checks(lib):
    L = lib.lib
    assert L.sq_weight_colmax(A, 1, 4, 24, A2, None) == lib.SQ_ERR_SHAPE
    assert L.sq_weight_colmax(A, 1, 4, 16, None, None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_weight_colmax(A, 5, 4, 16, A2, None) == lib.SQ_ERR_DTYPE
    assert L.sq_weight_colmax(MIS, 1, 4, 16, A2, None) == lib.SQ_ERR_ALIGN
    assert L.sq_smooth_scales_peaks(A, A, 16, 1.5, A2, A2, None, None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_smooth_scales_peaks(A, None, 16, 0.5, A2, A2, None, None) == \
        lib.SQ_ERR_INVALID_ARG
    assert L.sq_smooth_scales_peaks(A, A, 20, 0.5, A2, A2, None, None) == lib.SQ_ERR_SHAPE
    assert L.sq_smooth_scales_peaks(A, A, 16, 0.5, A2, A2, MIS, None) == lib.SQ_ERR_ALIGN


def test_gemm_bias_checks(lib):
    L = lib.lib
    assert L.sq_gemm_w8a8_bias(A, A, 4, 4, 16, A2, 1, A2, MIS, A2, 1, None, None, 0, None) == \
        lib.SQ_ERR_ALIGN
    assert L.sq_gemm_w8a8_bias(A, A, 4, 4, 24, A2, 1, A2, A2, A2, 1, None, None, 0, None) == \
        lib.SQ_ERR_SHAPE
    assert "sq_gemm_w8a8_bias" in lib.last_error()
    assert L.sq_gemm_w8a8_bias(A, A, 0, 4, 16, A2, 1, A2, A2, A2, 1, None, None, 0, None) == \
        lib.SQ_OK


def test_gemm_checks(lib):
    L = lib.lib
    assert L.sq_gemm_w8a8(A, A, 4, 4, 24, A2, 1, A2, A2, 1, None, None, 0, None) == \
        lib.SQ_ERR_SHAPE
    assert L.sq_gemm_w8a8(A, A, 4, 4, 16, A2, 1, A2, A2, 5, None, None, 0, None) == \
        lib.SQ_ERR_DTYPE
    assert L.sq_gemm_w8a8(A, None, 4, 4, 16, A2, 1, A2, A2, 1, None, None, 0, None) == \
        lib.SQ_ERR_INVALID_ARG
    assert L.sq_gemm_w8a8(A, A, 4, 4, 16, A2, 1, A2, MIS, 1, None, None, 0, None) == \
        lib.SQ_ERR_ALIGN
    assert L.sq_gemm_w8a8(A, A, 4, 4, 16, A2, 1, A2, A2, 1, MIS, None, 0, None) == \
        lib.SQ_ERR_ALIGN
    assert L.sq_gemm_w8a8(A, A, 0, 4, 16, A2, 1, A2, A2, 1, None, None, 0, None) == lib.SQ_OK
    assert L.sq_gemm_w8a8(A, A, 4, 0, 16, A2, 1, A2, A2, 1, None, None, 0, None) == lib.SQ_OK
    assert L.sq_gemm_workspace_bytes(0, 5, 16) == 0


def test_selftest_checks(lib):
    L = lib.lib
    assert L.sq_selftest_bounded_wait(0, None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_selftest_bounded_wait(2_000_000_000, None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_probe_mma_i8(0, 148, None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_probe_mma_i8((1 << 30) + 1, 148, None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_probe_mma_i8(16, 0, None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_probe_mma_i8_pair(0, 74, None) == lib.SQ_ERR_INVALID_ARG
    assert L.sq_probe_mma_i8_pair(16, 0, None) == lib.SQ_ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    """The product path has no fallback: a missing .so is an ImportError."""
    import importlib.util

    from w8a8_int8_gemm_calib_b200 import _lib as real

    spec = importlib.util.spec_from_file_location("sq_lib_copy", real.__file__)
    mod = importlib.util.module_from_spec(spec)
    monkeypatch.setattr(os.path, "exists", lambda p: False if p.endswith(".so") else True)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)


def test_gemm_decode_routing_on_the_host(lib):
    """Which GEMM shapes take the stream-K path (and so need scratch) is
    decided on the host; without a device the SM count is taken as 148.
    Up to 8 tokens always stream-K; 9-128 tokens only while the 128-row
    tiles across N would not give every SM one; more than 128 never.  The
    scratch size follows the header's formula."""
    f = lib.lib.sq_gemm_workspace_bytes
    sms = 148
    assert f(8, 49152, 12288) > 0
    assert f(16, 49152, 12288) == 0 and f(128, 49152, 12288) == 0  # 256 tiles of 192
    assert f(128, 12288, 12288) > 0                                  # 64 tiles
    assert f(16, 192 * (sms - 1), 4096) > 0                          # one tile short of the SMs
    assert f(129, 512, 4096) == 0
    # 1000 channels: 8 tile counters (256 bytes) + 148 SMs x 2 slots x 1 token x 128 x 4
    assert f(1, 1000, 12288) == 256 + sms * 2 * 1 * 128 * 4


def test_bounds_checked_build(lib):
    """The release library reports no bounds checks; the bounds-checked
    build (built here if it is missing) reports them and exports the same
    entry points."""
    import importlib.util

    assert lib.lib.sq_debug_bounds_enabled() == 0
    spec = importlib.util.spec_from_file_location(
        "sq_build", os.path.join(ROOT, "w8a8_int8_gemm_calib_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    path = b.LIB_DEBUG if os.path.exists(b.LIB_DEBUG) else b.build(debug_bounds=True)
    dbg = ctypes.CDLL(path)
    dbg.sq_debug_bounds_enabled.restype = ctypes.c_int
    assert dbg.sq_debug_bounds_enabled() == 1
    for n in declared_functions():
        assert hasattr(dbg, n), f"{n} missing from the bounds-checked build"
