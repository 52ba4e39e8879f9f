"""Failure detection without a GPU fault: a kernel waits on an mbarrier that
nothing arrives at, with a bounded wait; the wait runs out, the kernel
records SQ_ERR_TIMEOUT in the device status word and returns normally.
sq_sync_status() reports it once, clears it, and the context stays usable."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import w8a8_int8_gemm_calib_b200 as m

    return m


def test_bounded_wait_reports_timeout_and_context_survives(sq):
    sq.sq_sync_status()  # start clean
    sq.sq_selftest_bounded_wait(2_000_000)  # 2 ms limit on a wait that never completes
    with pytest.raises(sq.SQError) as ei:
        sq.sq_sync_status()
    assert ei.value.status == 7  # SQ_ERR_TIMEOUT
    sq.sq_sync_status()  # the word was cleared by the read above
    # the context still runs kernels correctly
    x = torch.randn(64, 256, device="cuda")
    amax = torch.zeros(256, device="cuda")
    sq.sq_calib_absmax(x, amax)
    sq.sq_sync_status()
    assert torch.equal(amax, x.abs().amax(dim=0))


def test_timeout_is_reported_once_per_fault(sq):
    for _ in range(2):
        sq.sq_selftest_bounded_wait(1_000)
        with pytest.raises(sq.SQError):
            sq.sq_sync_status()
    sq.sq_sync_status()
