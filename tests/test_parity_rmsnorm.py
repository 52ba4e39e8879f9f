"""GPU parity of the RMSNorm variants (NEXT-3: the fold gamma' = gamma / s
without a beta) against the CPU oracle, bit for bit: calibration peaks
through RMSNorm(x; gamma), the quantizer behind RMSNorm(x; gamma / s) at the
three granularities, and a whole smoothed linear with an RMSNorm in front.

Shapes cover the shared-memory row pipeline (fp32 register rows, rows in
storage form, every slice width) and the re-reading kernel for rows too wide
for it, both element types and ragged tails."""
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
    x = synth.activations(seed, f"rms{T}x{K}", T, K, out)
    return synth.bf16_bits(x) if dtype == "bf16" else x


def _gamma(seed, K):
    return synth.ln_params(seed, f"rmsg{K}", K)[0]


SHAPES = [(1, 16), (5, 48), (33, 1040), (130, 4096), (64, 5120), (9, 8192), (12, 12288),
          (3, 20480), (2, 53248)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,K", SHAPES)
def test_calib_absmax_rmsnorm(sq, orc, dtype, T, K):
    x = _x(T + 3 * K, T, K, dtype)
    g = _gamma(K, K)
    want = orc.calib_absmax_rms(x, g)
    amax = torch.zeros(K, dtype=torch.float32, device="cuda")
    sq.sq_calib_absmax_rms(dev(x), amax, dev(g))
    sq.sq_sync_status()
    assert_bits_equal(host(amax), want, "amax")
    x2 = _x(T + 5 * K, max(1, T // 2), K, dtype)
    sq.sq_calib_absmax_rms(dev(x2), amax, dev(g))
    sq.sq_sync_status()
    assert_bits_equal(host(amax), orc.calib_absmax_rms(x2, g, amax=want), "amax running")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("gran", ["token", "static", "tensor"])
@pytest.mark.parametrize("T,K", SHAPES)
def test_rms_smooth_quant_act(sq, orc, dtype, gran, T, K):
    x = _x(T + 7 * K, T, K, dtype)
    g = (_gamma(K + 1, K) / np.random.default_rng(K).uniform(0.2, 4.0, K)).astype(np.float32)
    kw = dict(per_token=gran == "token", per_tensor_dynamic=gran == "tensor")
    delta = np.float32(0.02)
    xq_want, act_want, ncl_want = orc.quant_act_rms(x, g, static_delta=delta, **kw)
    xq = torch.empty((T, K), dtype=torch.int8, device="cuda")
    if gran == "token":
        act = torch.empty(T, dtype=torch.float32, device="cuda")
    else:
        act = torch.full((1,), float(delta), dtype=torch.float32, device="cuda")
    ncl = torch.zeros(1, dtype=torch.int64, device="cuda")
    sq.sq_rms_smooth_quant_act(dev(x), xq, act, dev(g), n_clipped=ncl, **kw)
    sq.sq_sync_status()
    assert_bits_equal(host(xq), xq_want, "xq")
    assert_bits_equal(host(act), act_want, "act_scale")
    assert int(host(ncl)[0]) == ncl_want


def test_rmsnorm_linear_end_to_end(sq, orc):
    """The OPT-6.7B QKV shapes with an RMSNorm in front: calibration through
    RMSNorm(gamma), eq. (4), the fold (W * s, gamma / s with no beta), the
    quantizer behind RMSNorm(gamma / s), the GEMM -- every step bit-exact,
    the activations and outputs on sampled rows."""
    K, N, M, Tc = 4096, 12288, 2048, 4096
    out = synth.outlier_pattern(1001, K, count=12, tag="rmsk")
    x_cal = synth.bf16_bits(synth.activations(1001, "rms/x_cal", Tc, K, out))
    x = synth.bf16_bits(synth.activations(1001, "rms/x", M, K, out))
    w = synth.bf16_bits(synth.weights(1001, "rms/w", N, K, 0.02))
    g = _gamma(1001, K)
    o_amax = orc.calib_absmax_rms(x_cal, g)
    o_s, _ = orc.smooth_scales(o_amax, orc.weight_colmax(w), 0.5)
    o_wq, o_ws = orc.fuse_weights_q8(w, o_s)
    o_g2, _ = orc.fold_ln(g, None, o_s)
    rows = np.array([0, 1, 127, 128, 1024, M - 1], np.int64)
    o_xq, o_act, _ = orc.quant_act_rms(x[rows], o_g2, per_token=True)
    o_y, o_acc = orc.gemm_w8a8(o_xq, o_wq, o_act, o_ws, per_token=True, out_bf16=True)

    f32 = dict(dtype=torch.float32, device="cuda")
    amax = torch.zeros(K, **f32)
    sq.sq_calib_absmax_rms(dev(x_cal), amax, dev(g))
    s, inv_s = torch.empty(K, **f32), torch.empty(K, **f32)
    sq.sq_smooth_scales(amax, dev(w), 0.5, s, inv_s)
    wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    ws = torch.empty(N, **f32)
    g2 = torch.empty(K, **f32)
    sq.sq_fuse_weights_q8(dev(w), s, wq, ws, dev(g), None, g2, None)
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    act = torch.empty(M, **f32)
    sq.sq_rms_smooth_quant_act(dev(x), xq, act, g2)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    sq.sq_gemm_w8a8(xq, wq, act, ws, y, acc_out=acc, workspace=sq.Workspace())
    sq.sq_sync_status()
    assert_bits_equal(host(amax), o_amax, "amax")
    assert_bits_equal(host(s), o_s, "s")
    assert_bits_equal(host(ws), o_ws, "w_scale")
    assert_bits_equal(host(wq), o_wq, "wq")
    assert_bits_equal(host(g2), o_g2, "gamma/s")
    r = torch.from_numpy(rows).cuda()
    assert_bits_equal(host(xq[r]), o_xq, "xq rows")
    assert_bits_equal(host(act[r]), o_act, "act rows")
    assert_bits_equal(host(acc[r]), o_acc, "acc rows")
    assert_bits_equal(host(y[r]), o_y, "y rows")
