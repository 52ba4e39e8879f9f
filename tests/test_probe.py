"""The INT8 tensor-core rate probes (measurement support for the GEMM's
roofline): both launch forms run to completion without a time-out and
report an op count consistent with their arguments; a short launch's rate
is below the GPU's nominal dense INT8 rate at its maximum clock."""
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import w8a8_int8_gemm_calib_b200 as m

    return m


@pytest.mark.parametrize("pair", [False, True])
def test_probe_runs_and_counts(sq, pair):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    kblocks = 2000
    for _ in range(2):
        ops = (sq.sq_probe_mma_i8_pair(kblocks, sms // 2) if pair
               else sq.sq_probe_mma_i8(kblocks, sms))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    ops = (sq.sq_probe_mma_i8_pair(kblocks, sms // 2) if pair else sq.sq_probe_mma_i8(kblocks, sms))
    e1.record()
    sq.sq_sync_status()  # raises on a time-out
    assert ops == 8388608 * kblocks * sms - (8388608 * kblocks if pair and sms % 2 else 0)
    tops = ops / (e0.elapsed_time(e1) * 1e-3) / 1e12
    # 8192 int8 multiply-adds per clock per SM at 2 GHz bound any honest rate
    assert 0 < tops < 2 * 8192 * sms * 2.0e9 / 1e12
