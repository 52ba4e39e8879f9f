"""GPU parity of the fold of 1/s into a producing linear (NEXT-3; [review]
§5.5: the smoothing factor folds into the previous layer's parameters): the
producer's per-output-channel scale and bias divided by s, bit for bit
against the oracle, and a producer -> ReLU -> consumer chain in which the
consumer's quantizer takes no 1/s."""
import numpy as np
import pytest

import synth
from tests._util import assert_bits_equal, dev, host

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import w8a8_int8_gemm_calib_b200 as m

    return m


@pytest.mark.parametrize("K", [16, 1040, 5120, 20480])
@pytest.mark.parametrize("with_bias", [True, False])
def test_fold_into_producer(sq, orc, K, with_bias):
    r = np.random.default_rng(K)
    s = r.uniform(1e-4, 30.0, K).astype(np.float32)
    ws = r.uniform(1e-5, 1e-2, K).astype(np.float32)
    b = r.normal(0, 1, K).astype(np.float32) if with_bias else None
    ws_want, b_want = orc.fold_into_producer(s, ws, b)
    ws_d, b_d = dev(ws), dev(b)
    sq.sq_fold_into_producer(dev(s), ws_d, b_d)
    sq.sq_sync_status()
    assert_bits_equal(host(ws_d), ws_want, "w_scale")
    if with_bias:
        assert_bits_equal(host(b_d), b_want, "bias")


def test_producer_relu_consumer_chain(sq, orc):
    """fc1 (1024 -> 2048, bias) with the consumer's 1/s folded into its scale
    and bias, ReLU, then the consumer's per-token quantizer without 1/s: the
    codes and steps equal the oracle's same chain bit for bit."""
    T, Kin, K = 64, 1024, 2048
    r = np.random.default_rng(3)
    xq = r.integers(-127, 128, (T, Kin)).astype(np.int8)
    wq = r.integers(-127, 128, (K, Kin)).astype(np.int8)
    act = r.uniform(1e-3, 1e-2, T).astype(np.float32)
    ws = r.uniform(1e-5, 1e-3, K).astype(np.float32)
    b = r.normal(0, 0.5, K).astype(np.float32)
    s = r.uniform(0.05, 20.0, K).astype(np.float32)
    # oracle chain
    wsf, bf = orc.fold_into_producer(s, ws, b)
    y_bits, _ = orc.gemm_w8a8(xq, wq, act, wsf, out_bf16=True, bias=bf)
    relu = np.where(synth.bf16_bits_to_f32(y_bits) > 0, y_bits, np.uint16(0))
    xq2_want, act2_want, _ = orc.quant_act(relu, per_token=True)
    # GPU chain
    ws_d, b_d = dev(ws), dev(b)
    sq.sq_fold_into_producer(dev(s), ws_d, b_d)
    y = torch.empty((T, K), dtype=torch.bfloat16, device="cuda")
    sq.sq_gemm_w8a8(dev(xq), dev(wq), dev(act), ws_d, y, workspace=sq.Workspace(), bias=b_d)
    y = torch.relu(y)
    xq2 = torch.empty((T, K), dtype=torch.int8, device="cuda")
    act2 = torch.empty(T, dtype=torch.float32, device="cuda")
    sq.sq_ln_smooth_quant_act(y, xq2, act2)
    sq.sq_sync_status()
    assert_bits_equal(host(xq2), xq2_want, "consumer xq")
    assert_bits_equal(host(act2), act2_want, "consumer act_scale")
