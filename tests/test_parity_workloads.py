"""Parity at the full sizes of the five workloads, in the launch configuration
bench.py times: the whole path (calibration peak, eq. (4) factors, weight +
LayerNorm fold, activation quantizer, INT8 GEMM) on the GPU against the CPU
oracle on the same seeded inputs.

Compared bit for bit: the calibration peaks and smoothing factors (all K),
the weight scales and INT8 weights (all N x K), the static step, and -- on
sampled token rows (first, last, around a 128-row tile edge, and two seeded
random rows), every output column -- the INT8 activations, their scales and
the outputs.  For alpha outside {0, 0.5, 1}, where neither side's fp64 pow is
correctly rounded, the factors are compared within 1 fp32 ulp and the
downstream steps on both sides take the oracle's factors."""
import numpy as np
import pytest

import synth
from tests._util import assert_bits_equal, dev, host, ulp_diff_f32

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import w8a8_int8_gemm_calib_b200 as m

    return m


CASES = [(w, l.name) for w in synth.WORKLOAD_ORDER for l in synth.workloads()[w].linears]


def sample_rows(M, seed):
    r = np.random.default_rng(seed)
    rows = {0, 1, 127, 128, M // 2, M - 1, int(r.integers(0, M)), int(r.integers(0, M))}
    return np.array(sorted(x for x in rows if 0 <= x < M), dtype=np.int64)


@pytest.mark.parametrize("workload,linear", CASES)
def test_workload_parity(sq, orc, workload, linear):
    lin = next(l for l in synth.workloads()[workload].linears if l.name == linear)
    d = synth.make_linear_inputs(lin)
    K, N, M = lin.K, lin.N, lin.T
    f32 = dict(dtype=torch.float32, device="cuda")
    exact_alpha = lin.alpha in (0.0, 0.5, 1.0)

    # ---------------- oracle
    o_amax = orc.calib_absmax(d["x_cal"], d["gamma"], d["beta"], 1e-5)
    o_s, o_inv = orc.smooth_scales(o_amax, orc.weight_colmax(d["w"]), lin.alpha)
    o_dA = orc.static_delta(o_amax, o_s)
    o_wq, o_ws = orc.fuse_weights_q8(d["w"], o_s)
    rows = sample_rows(M, M + K)
    if lin.ln:
        o_g2, o_b2 = orc.fold_ln(d["gamma"], d["beta"], o_s)
        o_xq, o_act, _ = orc.quant_act(d["x"][rows], o_g2, o_b2, 1e-5,
                                       per_token=lin.per_token, static_delta=o_dA)
    else:
        o_xq, o_act, _ = orc.quant_act(d["x"][rows], inv_s=o_inv, per_token=lin.per_token,
                                       static_delta=o_dA)
    # oracle GEMM on the sampled rows only (act holds one entry per sampled row)
    o_y, o_acc = orc.gemm_w8a8(o_xq, o_wq, o_act, o_ws, per_token=lin.per_token,
                               out_bf16=(lin.dtype == "bf16"))

    # ---------------- GPU, the same calls bench.py makes
    x_cal, x, w = dev(d["x_cal"]), dev(d["x"]), dev(d["w"])
    g, b = dev(d["gamma"]), dev(d["beta"])
    amax = torch.zeros(K, **f32)
    sq.sq_calib_absmax(x_cal, amax, g, b, 1e-5)
    s, inv_s, dA = torch.empty(K, **f32), torch.empty(K, **f32), torch.empty(1, **f32)
    sq.sq_smooth_scales(amax, w, lin.alpha, s, inv_s, dA)
    sq.sq_sync_status()
    assert_bits_equal(host(amax), o_amax, "amax")
    if exact_alpha:
        assert_bits_equal(host(s), o_s, "s")
        assert_bits_equal(host(inv_s), o_inv, "inv_s")
        assert_bits_equal(host(dA), np.array([o_dA], np.float32), "delta_A")
    else:
        assert ulp_diff_f32(host(s), o_s).max() <= 1
        s.copy_(torch.from_numpy(o_s))
        inv_s.copy_(torch.from_numpy(o_inv))
        dA.fill_(float(o_dA))
    wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    ws = torch.empty(N, **f32)
    g2 = torch.empty(K, **f32) if lin.ln else None
    b2 = torch.empty(K, **f32) if lin.ln else None
    sq.sq_fuse_weights_q8(w, s, wq, ws, g, b, g2, b2)
    act = torch.empty(M, **f32) if lin.per_token else dA.clone()
    xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
    if lin.ln:
        sq.sq_ln_smooth_quant_act(x, xq, act, g2, b2, 1e-5, per_token=lin.per_token)
    else:
        sq.sq_ln_smooth_quant_act(x, xq, act, inv_s=inv_s, per_token=lin.per_token)
    y = torch.empty((M, N), dtype=torch.bfloat16 if lin.dtype == "bf16" else torch.float32,
                    device="cuda")
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    sq.sq_gemm_w8a8(xq, wq, act, ws, y, per_token=lin.per_token, acc_out=acc,
                    workspace=sq.Workspace())
    sq.sq_sync_status()

    assert_bits_equal(host(ws), o_ws, "w_scale")
    assert_bits_equal(host(wq), o_wq, "wq")
    if lin.ln:
        og2, ob2 = orc.fold_ln(d["gamma"], d["beta"], o_s)
        assert_bits_equal(host(g2), og2, "gamma/s")
        assert_bits_equal(host(b2), ob2, "beta/s")
    r = torch.from_numpy(rows).cuda()
    assert_bits_equal(host(xq[r]), o_xq, "xq rows")
    if lin.per_token:
        assert_bits_equal(host(act[r]), o_act, "act_scale rows")
    assert_bits_equal(host(acc[r]), o_acc, "acc rows")
    assert_bits_equal(host(y[r]), o_y, "y rows")
