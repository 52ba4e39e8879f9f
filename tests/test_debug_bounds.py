"""The bounds-checked build (build.py --debug-bounds, libsq_b200_debug.so):
every kernel checks the global-memory offsets it computes by hand, records
SQ_ERR_BOUNDS and skips an access outside its tensor.  No test here makes an
out-of-range access: the self-test checks an offset at a tensor's end
without touching memory, and the parity suites run unchanged on the
bounds-checked build -- ragged shapes, every kernel family -- where any
caught offset would surface as SQ_ERR_BOUNDS from sq_sync_status or as a
skipped store (a mismatch against the oracle)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DEBUG_LIB = os.path.join(ROOT, "w8a8_int8_gemm_calib_b200", "libsq_b200_debug.so")


@pytest.fixture(scope="module")
def debug_env():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    if not os.path.exists(DEBUG_LIB):
        subprocess.check_call([sys.executable, os.path.join(ROOT, "w8a8_int8_gemm_calib_b200",
                                                            "build.py"), "--debug-bounds"])
    return dict(os.environ, SQ_B200_LIB=DEBUG_LIB)


def test_release_build_records_nothing():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import w8a8_int8_gemm_calib_b200 as sq

    assert not sq.sq_debug_bounds_enabled()
    sq.sq_selftest_bounds_check()
    sq.sq_sync_status()  # no status recorded


def test_selftest_records_bounds(debug_env):
    code = ("import w8a8_int8_gemm_calib_b200 as sq\n"
            "assert sq.sq_debug_bounds_enabled()\n"
            "sq.sq_selftest_bounds_check()\n"
            "try:\n"
            "    sq.sq_sync_status()\n"
            "    raise SystemExit('no status recorded')\n"
            "except sq.SQError as e:\n"
            "    assert e.status == 9, e.status\n"
            "sq.sq_sync_status()  # cleared by the read\n"
            "print('bounds self-test OK')\n")
    r = subprocess.run([sys.executable, "-c", code], env=debug_env, cwd=ROOT,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]


def test_parity_suites_on_bounds_checked_build(debug_env):
    files = ["tests/test_parity_gemm.py", "tests/test_parity_rowops.py", "tests/test_parity_o2.py",
             "tests/test_parity_bmm.py", "tests/test_parity_rmsnorm.py"]
    r = subprocess.run([sys.executable, "-m", "pytest", *files, "-m", "gpu", "-x", "-q", "-p",
                        "no:cacheprovider"], env=debug_env, cwd=ROOT, capture_output=True,
                       text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]
