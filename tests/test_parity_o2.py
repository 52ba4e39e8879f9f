"""GPU parity of per-tensor dynamic activation quantization (the review's
SmoothQuant-O2, §6.3; dynamic steps §2.5) against the CPU oracle: one step
Delta(max over the whole call of |y|), computed in two passes over x on the
GPU.  Bit-exact: the step and every code.

Shapes cover the shared-memory row pipeline (one and two CTAs per SM, fp32
register rows, rows in storage form) and the re-reading row kernel for rows
too wide for it, with and without a LayerNorm, both element types, ragged
tails, a single token, an all-zero call and non-finite elements."""
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


def _x(seed, T, K, dtype, frac=0.01):
    out = synth.outlier_pattern(seed, K, frac)
    x = synth.activations(seed, f"o2x{T}x{K}", T, K, out)
    return synth.bf16_bits(x) if dtype == "bf16" else x


def _run(sq, x, g=None, b=None, inv=None):
    T, K = x.shape
    xq = torch.empty((T, K), dtype=torch.int8, device="cuda")
    act = torch.full((1,), 123.0, dtype=torch.float32, device="cuda")
    ncl = torch.zeros(1, dtype=torch.int64, device="cuda")
    sq.sq_ln_smooth_quant_act(dev(x), xq, act, dev(g), dev(b), 1e-5, dev(inv),
                              n_clipped=ncl, per_tensor_dynamic=True)
    sq.sq_sync_status()
    return host(xq), host(act), int(host(ncl)[0])


SHAPES = [(1, 16), (37, 48), (300, 1040), (129, 2064), (257, 4096), (64, 5120), (33, 8192),
          (16, 12288), (5, 20480), (3, 24576), (2, 53248)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", ["ln", "inv_s", "plain"])
@pytest.mark.parametrize("T,K", SHAPES)
def test_per_tensor_dynamic(sq, orc, dtype, mode, T, K):
    x = _x(T + K, T, K, dtype)
    g = b = inv = None
    if mode == "ln":
        g, b = synth.ln_params(K, f"o2ln{K}", K)
    elif mode == "inv_s":
        inv = np.random.default_rng(K).uniform(0.05, 2.0, K).astype(np.float32)
    xq_want, act_want, ncl_want = orc.quant_act(x, g, b, 1e-5, inv_s=inv, per_tensor_dynamic=True)
    xq, act, ncl = _run(sq, x, g, b, inv)
    assert_bits_equal(act, act_want, "act_scale")
    assert_bits_equal(xq, xq_want, "xq")
    assert ncl == ncl_want == 0


@pytest.mark.parametrize("mode", ["ln", "inv_s"])
def test_per_tensor_step_is_the_largest_token_step(sq, mode):
    """On the GPU alone: the per-tensor step equals the largest per-token step
    (Delta is monotone in the peak) and the codes equal static quantization
    with that step."""
    T, K = 1000, 4096
    x = dev(_x(5, T, K, "bf16"))
    g = b = inv = None
    if mode == "ln":
        g, b = [dev(v) for v in synth.ln_params(3, "o2rel", K)]
    else:
        inv = dev(np.random.default_rng(2).uniform(0.05, 2.0, K).astype(np.float32))
    xq2 = torch.empty((T, K), dtype=torch.int8, device="cuda")
    act2 = torch.empty(1, dtype=torch.float32, device="cuda")
    sq.sq_ln_smooth_quant_act(x, xq2, act2, g, b, 1e-5, inv, per_tensor_dynamic=True)
    xq1 = torch.empty_like(xq2)
    act1 = torch.empty(T, dtype=torch.float32, device="cuda")
    sq.sq_ln_smooth_quant_act(x, xq1, act1, g, b, 1e-5, inv, per_token=True)
    xq3 = torch.empty_like(xq2)
    sq.sq_ln_smooth_quant_act(x, xq3, act2.clone(), g, b, 1e-5, inv, per_token=False)
    sq.sq_sync_status()
    assert act2.item() == act1.max().item()
    assert torch.equal(xq2, xq3)
    assert int(xq2.abs().max()) == 127


def test_per_tensor_dynamic_edges(sq, orc):
    """All-zero call (the step floor), NaN elements (skipped by the peak,
    coded 0) and an infinite element (infinite step, every code 0)."""
    z = np.zeros((7, 64), np.float32)
    xq, act, _ = _run(sq, z)
    assert act[0] == np.float32(np.float32(1e-7) / np.float32(127)) and not xq.any()
    x = _x(11, 9, 1024, "f32")
    x[2, 5] = np.nan
    x[7, 900] = np.nan
    for case in ("nan", "inf"):
        if case == "inf":
            x[4, 17] = np.inf
        xq_want, act_want, _ = orc.quant_act(x, per_tensor_dynamic=True)
        xq, act, _ = _run(sq, x)
        assert_bits_equal(act, act_want, f"act_scale ({case})")
        assert_bits_equal(xq, xq_want, f"xq ({case})")


def test_per_tensor_dynamic_feeds_the_gemm(sq, orc):
    """The O2 step drives the GEMM's per-tensor dequantization: outputs
    bit-exact against the oracle on sampled rows."""
    T, K, N = 300, 1040, 272
    x = _x(21, T, K, "bf16")
    wq = np.random.default_rng(4).integers(-127, 128, (N, K)).astype(np.int8)
    ws = np.random.default_rng(5).uniform(1e-4, 1e-2, N).astype(np.float32)
    xq_want, act_want, _ = orc.quant_act(x, per_tensor_dynamic=True)
    rows = np.array([0, 1, 127, 128, 299], np.int64)
    y_want, acc_want = orc.gemm_w8a8(xq_want, wq, act_want, ws, per_token=False, rows=rows,
                                     out_bf16=True)
    xq = torch.empty((T, K), dtype=torch.int8, device="cuda")
    act = torch.empty(1, dtype=torch.float32, device="cuda")
    sq.sq_ln_smooth_quant_act(dev(x), xq, act, per_tensor_dynamic=True)
    y = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    acc = torch.empty((T, N), dtype=torch.int32, device="cuda")
    sq.sq_gemm_w8a8(xq, dev(wq), act, dev(ws), y, per_token=False, acc_out=acc,
                    workspace=sq.Workspace())
    sq.sq_sync_status()
    r = torch.from_numpy(rows).cuda()
    assert_bits_equal(host(acc[r]), acc_want, "acc")
    assert_bits_equal(host(y[r]), y_want, "y")
