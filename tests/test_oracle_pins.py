"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test pins one oracle function to something other than itself: a value
the pages print, a closed form, an invariant, a textbook special case, a
library routine, or brute force on tiny inputs.

Sources:
* [explainer] "SmoothQuant 如何解决激活量化难题？为什么适合 W8A8？"
* [review]    "SmoothQuant：大型语言模型的精准高效训练后量化 — 深度技术评审"
* [embedded]  "嵌入式 SLM 动态权重量化：SmoothQuant 激活异常值迁移与 INT8 部署实战"
"""
import json
import math
import os

import numpy as np
import pytest

import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")
F32_EPS = np.finfo(np.float32).eps


def ulps(a, b):
    """Distance in fp32 ulps (of the larger magnitude)."""
    a = np.float64(a)
    b = np.float64(b)
    m = max(abs(a), abs(b))
    if m == 0:
        return 0.0
    ulp = np.spacing(np.float32(m))
    return abs(a - b) / float(ulp)


# ------------------------------------------------------------------ P-1 / P-2

def test_worked_example_s10(orc):
    """[explainer] §三: peaks 120 and 0.12 with a chosen s = 10 become 12 and
    1.2, and the float product is unchanged."""
    g = json.load(open(os.path.join(GOLD, "worked_example.json")))
    K = 16
    # calibration activations: channel 0 peaks at -120 (sign must not matter)
    xc = np.ones((4, K), np.float32) * 0.5
    xc[2, 0] = -g["act_peak"]
    xc[1, 0] = 3.0
    amax = orc.calib_absmax(xc)
    assert amax[0] == np.float32(g["act_peak"])
    s = np.ones(K, np.float32)
    s[0] = g["s"]
    # static scale: the smoothed activation peak is exactly 12
    dA = orc.static_delta(amax, s)
    assert dA == np.float32(np.float32(g["act_peak_smoothed"]) / np.float32(127.0))
    # a weight matrix whose channel-0 peak is 0.12 (row 3)
    w = np.full((5, K), 0.01, np.float32)
    w[3, 0] = g["w_peak"]
    wq, ws = orc.fuse_weights_q8(w, s)
    w_hat_peak = np.float64(ws[3]) * 127.0
    assert ulps(w_hat_peak, g["w_peak_smoothed"]) <= 2
    # the peak element lands on the top code; others scale down accordingly
    assert wq[3, 0] == 127
    # product preserved: (120/10) * (0.12*10) == 120*0.12 == 14.4
    prod = np.float64(dA) * 127.0 * w_hat_peak
    assert abs(prod - g["act_peak"] * g["w_peak"]) / 14.4 < 4 * F32_EPS
    # and the peak activation quantizes to the top code under that scale
    xq, _, ncl = orc.quant_act(xc, inv_s=(1.0 / s).astype(np.float32),
                               per_token=False, static_delta=dA)
    assert xq[2, 0] == -127 and ncl == 0


def test_eq4_alpha_half_closed_form(orc):
    """[review] §5.3 eq. (4) at alpha = 0.5 on the worked-example peaks."""
    g = json.load(open(os.path.join(GOLD, "worked_example.json")))["alpha_half"]
    s, inv_s = orc.smooth_scales(np.array([120.0], np.float32),
                                 np.array([0.12], np.float32), 0.5)
    assert ulps(s[0], g["s"]) <= 1
    assert ulps(np.float32(120.0) / s[0], g["smoothed_peak"]) <= 2
    assert ulps(np.float32(0.12) * s[0], g["smoothed_peak"]) <= 2
    assert inv_s[0] == np.float32(1.0) / s[0]


def test_eq4_alpha_half_balances_peaks(orc):
    """eq. (4) at alpha = 0.5: max|X_hat_j| = max|W_hat_j| = sqrt(a*b)."""
    r = np.random.default_rng(1)
    a = r.uniform(0.01, 200, 512).astype(np.float32)
    b = r.uniform(1e-3, 0.5, 512).astype(np.float32)
    s, _ = orc.smooth_scales(a, b, 0.5)
    for j in range(512):
        ref = math.sqrt(float(a[j]) * float(b[j]))
        assert ulps(a[j] / s[j], ref) <= 2
        assert ulps(b[j] * s[j], ref) <= 2
        assert ulps(s[j], math.sqrt(float(a[j]) / float(b[j]))) <= 0.5 + 1e-9


def test_eq4_general_alpha_closed_form(orc):
    """eq. (4) for alpha outside {0, 0.5, 1} against an fp64 evaluation of
    exp(alpha*ln a - (1-alpha)*ln b) (a different route than pow/pow):
    within 1 fp32 ulp (the unpinned remainder is pow's own rounding)."""
    r = np.random.default_rng(2)
    a = r.uniform(0.01, 200, 256).astype(np.float32)
    b = r.uniform(1e-3, 0.5, 256).astype(np.float32)
    for alpha in (0.25, 0.75, 0.8, 0.4):
        s, _ = orc.smooth_scales(a, b, alpha)
        al = float(np.float32(alpha))  # alpha is an fp32 argument
        for j in range(256):
            ref = math.exp(al * math.log(float(a[j])) -
                           (1 - al) * math.log(float(b[j])))
            assert ulps(s[j], ref) <= 1.0


# ------------------------------------------------------------------ P-4 / P-5

def test_alpha_one_flattens_activation_peaks(orc):
    """alpha = 1: every smoothed activation channel's absmax equals 1
    ([embedded] §一.2; [review] §5.3)."""
    lin = synth.workloads()["tiny_k1024"].linears[0]
    d = synth.make_linear_inputs(lin, T=64, T_cal=96, N=32)
    amax = orc.calib_absmax(d["x_cal"])
    aw = orc.weight_colmax(d["w"])
    s, inv_s = orc.smooth_scales(amax, aw, 1.0)
    assert np.array_equal(s, np.maximum(amax, np.float32(1e-4)))
    # exact division path: the static scale is exactly delta(1)
    assert orc.static_delta(amax, s) == np.float32(1.0) / np.float32(127.0)
    # multiply-by-reciprocal path: within 2 ulp of 1
    xs = d["x_cal"] * inv_s[None, :]
    pk = np.abs(xs).max(axis=0)
    assert np.all(np.abs(pk.astype(np.float64) - 1.0) <= 2 * F32_EPS)


def test_alpha_zero_normalises_weight_channels(orc):
    """alpha = 0: s_j = 1/max|W_j|, so every scaled weight input channel has
    absmax 1 (eq. (4) with alpha = 0)."""
    r = np.random.default_rng(3)
    w = (r.standard_normal((48, 64)) * 0.02).astype(np.float32)
    aw = orc.weight_colmax(w)
    amax = r.uniform(0.5, 100, 64).astype(np.float32)
    s, _ = orc.smooth_scales(amax, aw, 0.0)
    pk = np.abs(w * s[None, :]).max(axis=0)
    assert np.all(np.abs(pk.astype(np.float64) - 1.0) <= F32_EPS)


def test_scale_guards(orc):
    """Zero activation peak -> s floored at 1e-4; zero weight column -> the
    1e-7 floor keeps s finite ([embedded] §三 guards)."""
    s, inv = orc.smooth_scales(np.array([0.0, 5.0, 0.0], np.float32),
                               np.array([0.3, 0.0, 0.0], np.float32), 0.5)
    assert s[0] == np.float32(1e-4)
    assert np.isfinite(s[1]) and ulps(s[1], math.sqrt(5.0 / float(np.float32(1e-7)))) <= 1
    assert s[2] == np.float32(1e-4)
    assert np.all(np.isfinite(inv))


# ------------------------------------------------------------------ P-3

def test_fold_preserves_the_linear_map(orc):
    """eq. (3) ([review] §5.1): (X diag(s)^-1)(diag(s) W) = XW.  The oracle's
    LayerNorm fold (gamma/s, beta/s) and weight fold (W*s), composed in fp64,
    reproduce the unfolded LN(X) W^T to fp32 rounding."""
    lin = synth.workloads()["tiny_k1024"].linears[0]
    d = synth.make_linear_inputs(lin, T=8, T_cal=64, N=16)
    amax = orc.calib_absmax(d["x_cal"], d["gamma"], d["beta"])
    s, _ = orc.smooth_scales(amax, orc.weight_colmax(d["w"]), 0.5)
    g2, b2 = orc.fold_ln(d["gamma"], d["beta"], s)
    w64 = d["w"].astype(np.float64)
    for t in range(8):
        y = orc.layernorm_row(d["x"][t], d["gamma"], d["beta"]).astype(np.float64)
        yh = orc.layernorm_row(d["x"][t], g2, b2).astype(np.float64)
        ref = w64 @ y
        got = (w64 * s.astype(np.float64)[None, :]) @ yh
        rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert rel < 2e-6, rel


def test_eq3_identity_fp64():
    """eq. (3) itself in fp64 on outlier-structured data: 1e-13 relative."""
    r = np.random.default_rng(4)
    X = r.standard_normal((32, 96))
    X[:, [5, 60]] *= 90.0
    W = r.standard_normal((96, 40)) * 0.02
    s = r.uniform(0.1, 30.0, 96)
    lhs = (X / s[None, :]) @ (s[:, None] * W)
    rhs = X @ W
    assert np.linalg.norm(lhs - rhs) / np.linalg.norm(rhs) <= 1e-13


def test_end_to_end_error_bound(orc):
    """The W8A8 output stays within the quantization error bound of the fp64
    product of the smoothed operands: per element,
    |Y - sum_k xh_k wh_k| <= sum_k (|xh_k| dw/2 + |wh_k| dx/2 + dx dw/4)
    plus fp32 slack.  A dropped scale, a transposed operand or a sign error
    breaks it by orders of magnitude."""
    lin = synth.workloads()["tiny_k1024"].linears[0]
    d = synth.make_linear_inputs(lin, T=12, T_cal=64, N=24)
    amax = orc.calib_absmax(d["x_cal"])
    s, inv_s = orc.smooth_scales(amax, orc.weight_colmax(d["w"]), 0.5)
    wq, ws = orc.fuse_weights_q8(d["w"], s)
    xq, act, _ = orc.quant_act(d["x"], inv_s=inv_s, per_token=True)
    y, acc = orc.gemm_w8a8(xq, wq, act, ws, per_token=True)
    xh = d["x"].astype(np.float64) * inv_s.astype(np.float64)[None, :]
    wh = d["w"].astype(np.float64) * s.astype(np.float64)[None, :]
    ref = xh @ wh.T
    dx = act.astype(np.float64)[:, None]
    dw = ws.astype(np.float64)[None, :]
    bound = (np.abs(xh) @ np.ones((xh.shape[1], 1))) * dw / 2 \
        + dx / 2 * (np.abs(wh).sum(axis=1))[None, :] + xh.shape[1] * dx * dw / 4
    err = np.abs(y.astype(np.float64) - ref)
    assert np.all(err <= bound * 1.001 + 1e-6 * np.abs(ref))
    # and the bound is not vacuous: the result tracks the reference closely
    assert np.linalg.norm(err) / np.linalg.norm(ref) < 0.05


# ------------------------------------------------------------------ P-6 GEMM

def test_gemm_brute_force_tiny(orc):
    """Tiny GEMMs against Python-integer triple loops, including the int8
    extremes; dequantization against an fp64 product rounded once."""
    r = np.random.default_rng(5)
    for (M, N, K) in [(1, 1, 16), (3, 5, 32), (17, 13, 64), (7, 17, 48)]:
        xq = r.integers(-127, 128, (M, K)).astype(np.int8)
        wq = r.integers(-127, 128, (N, K)).astype(np.int8)
        xq[0, :] = 127
        wq[0, :] = -127
        act = r.uniform(1e-3, 1.0, M).astype(np.float32)
        ws = r.uniform(1e-4, 1e-2, N).astype(np.float32)
        y, acc = orc.gemm_w8a8(xq, wq, act, ws, per_token=True)
        for t in range(M):
            for n in range(N):
                ref = 0
                for k in range(K):
                    ref += int(xq[t, k]) * int(wq[n, k])
                assert acc[t, n] == ref
                # y = (float)acc * (as*ws): the product of two fp32 values is
                # exact in fp64, so one rounding of it must reproduce y
                scale = np.float32(np.float64(act[t]) * np.float64(ws[n]))
                yref = np.float32(np.float64(np.float32(ref)) * np.float64(scale))
                assert y[t, n] == yref


def test_gemm_bias_exact(orc):
    """The bias is added after the dequantization, per output channel
    ([review] §5.1 eq. (3): smoothing leaves a linear's bias untouched).  With
    power-of-two scales (2^-3 x 2^-5) and biases on the same 2^-8 grid every
    value is exact in fp32, so y = (acc + j) / 256 for bias[n] = j / 256 --
    checked against Python integers; a zero bias changes nothing."""
    r = np.random.default_rng(15)
    M, N, K = 9, 13, 64
    xq = r.integers(-127, 128, (M, K)).astype(np.int8)
    wq = r.integers(-127, 128, (N, K)).astype(np.int8)
    act = np.full(M, 2.0 ** -3, np.float32)
    ws = np.full(N, 2.0 ** -5, np.float32)
    j = r.integers(-1000, 1001, N)
    bias = (j / 256.0).astype(np.float32)
    y, acc = orc.gemm_w8a8(xq, wq, act, ws, per_token=True, bias=bias)
    for t in range(M):
        for n in range(N):
            ref = sum(int(xq[t, k]) * int(wq[n, k]) for k in range(K))
            assert acc[t, n] == ref
            assert y[t, n] == np.float32((ref + int(j[n])) / 256.0)
    y0, _ = orc.gemm_w8a8(xq, wq, act, ws, per_token=True, bias=np.zeros(N, np.float32))
    y1, _ = orc.gemm_w8a8(xq, wq, act, ws, per_token=True)
    assert np.array_equal(y0, y1)


def test_bmm_brute_force_tiny(orc):
    """The batched form (attention's INT8 matmuls, [review] §5.6 Fig. 6):
    every batch against Python-integer triple loops and a once-rounded fp64
    dequantization, with per-token / per-tensor activation steps and
    per-channel / per-batch weight steps; a scale taken from the wrong batch
    or axis fails."""
    r = np.random.default_rng(17)
    B, M, N, K = 3, 5, 7, 48
    xq = r.integers(-127, 128, (B, M, K)).astype(np.int8)
    wq = r.integers(-127, 128, (B, N, K)).astype(np.int8)
    for per_token in (True, False):
        for per_channel in (True, False):
            act = r.uniform(1e-3, 1.0, B * M if per_token else B).astype(np.float32)
            ws = r.uniform(1e-4, 1e-2, B * N if per_channel else B).astype(np.float32)
            y, acc = orc.bmm_w8a8(xq, wq, act, ws, per_token, per_channel)
            for b in range(B):
                for t in range(M):
                    for n in range(N):
                        ref = sum(int(xq[b, t, k]) * int(wq[b, n, k]) for k in range(K))
                        assert acc[b, t, n] == ref
                        a = act[b * M + t] if per_token else act[b]
                        w = ws[b * N + n] if per_channel else ws[b]
                        scale = np.float32(np.float64(a) * np.float64(w))
                        assert y[b, t, n] == np.float32(np.float64(np.float32(ref)) * scale)


def test_gemm_saturation_closed_form(orc):
    """All-127 operands: acc = 127*127*K = 16129*K (K=20480 -> 330,321,920),
    the largest magnitude any layer in the workloads reaches."""
    K = 20480
    xq = np.full((2, K), 127, np.int8)
    wq = np.full((3, K), 127, np.int8)
    wq[1] = -127
    y, acc = orc.gemm_w8a8(xq, wq, np.ones(1, np.float32), np.ones(3, np.float32),
                           per_token=False)
    assert acc[0, 0] == 330321920 and acc[1, 1] == -330321920


def test_gemm_rows_and_bf16(orc):
    """Sampled rows reproduce the full result; bf16 output = RNE of fp32."""
    r = np.random.default_rng(6)
    M, N, K = 9, 11, 80
    xq = r.integers(-127, 128, (M, K)).astype(np.int8)
    wq = r.integers(-127, 128, (N, K)).astype(np.int8)
    act = r.uniform(1e-3, 1.0, M).astype(np.float32)
    ws = r.uniform(1e-4, 1e-2, N).astype(np.float32)
    yf, acc = orc.gemm_w8a8(xq, wq, act, ws)
    rows = np.array([8, 0, 4])
    yr, accr = orc.gemm_w8a8(xq, wq, act, ws, rows=rows)
    assert np.array_equal(accr, acc[rows]) and np.array_equal(yr, yf[rows])
    yb, _ = orc.gemm_w8a8(xq, wq, act, ws, out_bf16=True)
    assert np.array_equal(yb, _torch_bf16_bits(yf))
    ref = xq.astype(np.int64) @ wq.astype(np.int64).T
    assert np.array_equal(acc, ref)


# ------------------------------------------------------------------ P-7 quantizer

def test_quantizer_ties_and_bounds(orc):
    """[review] §2.2: X_int8 = round(X/delta), delta = max|X|/127; ties go to
    even, the range is the symmetric [-127, 127]."""
    d = 0.25  # a power of two: v/d is exact
    assert orc.quant(0.5 * d, d) == 0
    assert orc.quant(1.5 * d, d) == 2
    assert orc.quant(2.5 * d, d) == 2
    assert orc.quant(-2.5 * d, d) == -2
    assert orc.quant(-0.5 * d, d) == 0
    assert orc.quant(126.5 * d, d) == 126
    assert orc.quant(127.5 * d, d) == 127       # saturates, not 128
    assert orc.quant(-1000.0, d) == -127        # never -128
    assert orc.quant(float("inf"), d) == 127
    assert orc.quant(float("-inf"), d) == -127
    assert orc.quant(float("nan"), d) == 0
    # the peak maps to the top code; error within half a step elsewhere
    r = np.random.default_rng(7)
    v = r.standard_normal(4096).astype(np.float32) * 3
    dd = orc.delta(float(np.abs(v).max()))
    q = np.array([orc.quant(float(t), dd) for t in v])
    assert q[np.argmax(np.abs(v))] in (127, -127)
    assert np.all(np.abs(v.astype(np.float64) - dd * q) <= dd / 2 * (1 + 1e-6))


def test_delta_floor(orc):
    assert orc.delta(0.0) == np.float32(np.float32(1e-7) / np.float32(127.0))
    assert orc.delta(127.0) == np.float32(1.0)
    xq, act, _ = orc.quant_act(np.zeros((3, 32), np.float32), per_token=True)
    assert not xq.any() and np.all(act == np.float32(np.float32(1e-7) / np.float32(127)))


def test_per_token_quant_properties(orc):
    """Per-token dynamic quantization ([review] §2.5, §6.3 O1): every row's
    peak maps to +-127 and every code is within half a step."""
    lin = synth.workloads()["tiny_k1024"].linears[0]
    d = synth.make_linear_inputs(lin, T=16, T_cal=32, N=8)
    inv_s = np.random.default_rng(8).uniform(0.05, 2, 1024).astype(np.float32)
    xq, act, ncl = orc.quant_act(d["x"], inv_s=inv_s, per_token=True)
    y = d["x"] * inv_s[None, :]
    assert ncl == 0
    for t in range(16):
        assert act[t] == orc.delta(float(np.abs(y[t]).max()))
        assert np.abs(xq[t]).max() == 127
        err = np.abs(y[t].astype(np.float64) - np.float64(act[t]) * xq[t])
        assert np.all(err <= act[t] / 2 * (1 + 1e-5))


def test_static_quant_saturates(orc):
    """Static per-tensor scale ([review] §2.5, §6.3 O3): runtime values above
    the calibrated peak saturate to +-127 and are counted."""
    x = np.array([[1.0, -1.0, 3.0, -5.0] * 4], np.float32)
    xq, _, ncl = orc.quant_act(x, per_token=False, static_delta=np.float32(1.0 / 64))
    assert xq[0, 0] == 64 and xq[0, 1] == -64
    assert xq[0, 2] == 127 and xq[0, 3] == -127
    assert ncl == 8


def test_per_tensor_dynamic_hand_example(orc):
    """Per-tensor dynamic quantization ([review] §6.3 O2; dynamic steps §2.5):
    one step from the peak of the whole call.  Peak 4 -> Delta = 4/127, 1/Delta
    = 31.75 (to fp32), so 1 -> 31.75 -> 32, -3 -> -95.25 -> -95, 1.5 -> 47.625
    -> 48, 4 -> 127, 0.25 -> 7.9375 -> 8, -1 -> -32, 0.5 -> 15.875 -> 16.  The
    peak lies in the second row: a per-row step would code the first row
    differently."""
    x = np.array([[1.0, -3.0, 0.0, 1.5], [4.0, 0.25, -1.0, 0.5]], np.float32)
    xq, act, ncl = orc.quant_act(x, per_tensor_dynamic=True)
    assert act.shape == (1,) and act[0] == np.float32(4.0) / np.float32(127.0)
    assert xq.tolist() == [[32, -95, 0, 48], [127, 8, -32, 16]]
    assert ncl == 0
    xq1, act1, _ = orc.quant_act(x, per_token=True)
    assert xq1[0].tolist() != xq[0].tolist()  # row 0 alone peaks at 3


def test_per_tensor_dynamic_relations(orc):
    """O2 against O1 and O3 on outlier-structured data, with and without a
    LayerNorm: Delta is monotone in the peak, so the per-tensor step equals
    the largest per-token step exactly, the codes equal static quantization
    with that step, the global peak maps to +-127, and a one-row call equals
    per-token quantization."""
    lin = synth.workloads()["tiny_k1024"].linears[0]
    d = synth.make_linear_inputs(lin, T=24, T_cal=32, N=8)
    rng = np.random.default_rng(21)
    inv_s = rng.uniform(0.05, 2, 1024).astype(np.float32)
    g = (1 + 0.1 * rng.standard_normal(1024)).astype(np.float32)
    b = (0.02 * rng.standard_normal(1024)).astype(np.float32)
    for kw in (dict(inv_s=inv_s), dict(gamma_s=g, beta_s=b)):
        xq2, act2, ncl2 = orc.quant_act(d["x"], per_tensor_dynamic=True, **kw)
        _, act1, _ = orc.quant_act(d["x"], per_token=True, **kw)
        assert act2[0] == act1.max()
        xq3, _, ncl3 = orc.quant_act(d["x"], per_token=False, static_delta=act2[0], **kw)
        assert np.array_equal(xq2, xq3) and ncl2 == ncl3 == 0
        assert np.abs(xq2).max() == 127
        t_peak = int(np.argmax(act1))
        assert np.abs(xq2[t_peak]).max() == 127
        xq_one, act_one, _ = orc.quant_act(d["x"][5:6], per_tensor_dynamic=True, **kw)
        xq_tok, act_tok, _ = orc.quant_act(d["x"][5:6], per_token=True, **kw)
        assert act_one[0] == act_tok[0] and np.array_equal(xq_one, xq_tok)


def test_per_tensor_dynamic_non_finite(orc):
    """NaN elements are skipped by the peak and coded 0; an infinite element
    makes the step infinite, so every finite element codes to 0.  Peak 2:
    1/Delta rounds to exactly 63.5 in fp32, so 1 -> 63.5 -> 64 (tie to even)
    and -2 -> -127."""
    x = np.array([[1.0, np.nan, -2.0, 0.5], [0.25, 1.0, np.nan, -1.0]], np.float32)
    xq, act, _ = orc.quant_act(x, per_tensor_dynamic=True)
    assert act[0] == np.float32(2.0) / np.float32(127.0)
    assert xq[0, 1] == 0 and xq[1, 2] == 0 and xq[0, 2] == -127 and xq[0, 0] == 64
    x[1, 0] = np.inf
    xq, act, _ = orc.quant_act(x, per_tensor_dynamic=True)
    assert np.isinf(act[0]) and not xq.any()


def _torch_bf16_bits(v):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_bf16_rounding_matches_library(orc):
    """fp32 -> bf16 RNE against torch's conversion, including exact ties and
    NaN (the oracle's and the input generator's casts both)."""
    r = np.random.default_rng(9)
    v = r.standard_normal(3000).astype(np.float32) * 10
    ties = (np.arange(64, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    v = np.concatenate([v, ties, np.array([0.0, -0.0, 1e-40, 3.4e38], np.float32)])
    want = _torch_bf16_bits(v)
    assert np.array_equal(orc.f32_to_bf16_bits(v), want)
    assert np.array_equal(synth.bf16_bits(v), want)
    nan = orc.f32_to_bf16_bits(np.array([np.nan], np.float32))
    assert (nan[0] & 0x7F80) == 0x7F80 and (nan[0] & 0x7F) != 0


# ------------------------------------------------------------------ P-8 LN

def test_layernorm_matches_fp64(orc):
    """Canonical-order LayerNorm against an fp64 two-pass LayerNorm."""
    r = np.random.default_rng(10)
    for K in (16, 48, 1040, 4096, 5120):
        x = r.standard_normal(K).astype(np.float32)
        x[r.integers(0, K, 3)] *= 80
        g = (1 + 0.1 * r.standard_normal(K)).astype(np.float32)
        b = (0.02 * r.standard_normal(K)).astype(np.float32)
        y = orc.layernorm_row(x, g, b)
        x64 = x.astype(np.float64)
        mu = x64.mean()
        var = ((x64 - mu) ** 2).mean()
        ref = (x64 - mu) / np.sqrt(var + 1e-5) * g + b
        assert np.max(np.abs(y - ref)) <= 1e-5 * max(1.0, np.abs(ref).max())


def test_layernorm_exact_on_integer_rows(orc):
    """Integer rows with power-of-two length: every partial sum is exact, so
    mean and variance are exact whatever the order, and the output equals the
    closed form evaluated with those exact moments."""
    K = 1024
    x = np.tile(np.array([-3.0, -1.0, 1.0, 3.0], np.float32), K // 4)
    g = np.ones(K, np.float32)
    y = orc.layernorm_row(x, g, None, eps=0.0)
    # mean 0, variance 5 exactly
    rstd = np.float32(1.0) / np.sqrt(np.float32(5.0))
    assert np.array_equal(y, (x * rstd).astype(np.float32))


def test_rmsnorm_matches_fp64(orc):
    """Canonical-order RMSNorm against an fp64 RMSNorm (the norm of models
    whose smoothing fold is gamma / s alone)."""
    r = np.random.default_rng(12)
    for K in (16, 48, 1040, 4096, 5120):
        x = r.standard_normal(K).astype(np.float32)
        x[r.integers(0, K, 3)] *= 80
        g = (1 + 0.1 * r.standard_normal(K)).astype(np.float32)
        y = orc.rmsnorm_row(x, g)
        x64 = x.astype(np.float64)
        ref = x64 / np.sqrt((x64 ** 2).mean() + 1e-5) * g
        assert np.max(np.abs(y - ref)) <= 1e-5 * max(1.0, np.abs(ref).max())


def test_rmsnorm_exact_closed_form(orc):
    """Rows of +-2 with eps = 0: the mean of squares is exactly 4 in any
    order, rstd = 1/2 exactly, so y = +-gamma exactly; a mean term (the
    LayerNorm's) would make the +-2 pattern with a non-zero mean differ."""
    K = 1024
    r = np.random.default_rng(13)
    x = np.where(r.random(K) < 0.7, 2.0, -2.0).astype(np.float32)
    g = (1 + 0.1 * r.standard_normal(K)).astype(np.float32)
    y = orc.rmsnorm_row(x, g, eps=0.0)
    assert np.array_equal(y, np.where(x > 0, g, -g).astype(np.float32))
    assert not np.array_equal(orc.layernorm_row(x, g, None, eps=0.0), y)


# Rows whose fp32 mean depends on the order of the canonical reduction: two
# elements of +-2^24 and two ones.  Under the library's order the pair that
# is summed first decides whether a one is lost to rounding (2^24 + 1 is a
# tie and rounds to the even 2^24; -2^24 + 1 is exact).
#
# Row A (the cross-group combination): 2^24 at k = 0 (slot 0, group 0),
# -2^24 at k = 256 (slot 32, group 1), 1 at k = 512 (group 2) and k = 768
# (group 3).  Each group's butterfly only adds zeros to its one element, so
# (r0, r1, r2, r3) = (2^24, -2^24, 1, 1) and (r0 + r2) + (r1 + r3) =
# 2^24 + (-2^24 + 1) = 1.  Left to right, or (r0 + r1) + (r2 + r3), gives 2.
#
# Row B (the butterfly inside a group): 2^24 at k = 0 (slot 0), -2^24 at
# k = 8 (slot 1), 1 at k = 128 (slot 16) and k = 136 (slot 17).  The first
# butterfly round (xor 16) pairs slot 0 with 16 and slot 1 with 17: 2^24 and
# -2^24 + 1; the last round (xor 1) adds those: 1.  A butterfly starting at
# xor 1, or a sequential sum, gives 0 + 2 = 2.
#
# Either way mu = 1/1024 = 2^-10 exactly.  Variance pass: (+-2^24 - mu)
# rounds to +-2^24, whose square 2^48 absorbs every other term of its slot
# and group (each < 2^24, half an ulp of 2^48); the two 2^48 meet in the
# final sum, so var = 2^49 / 1024 = 2^39 in both rows.
def _order_rows():
    K = 1024
    a = np.zeros(K, np.float32)
    a[0], a[256], a[512], a[768] = 2.0 ** 24, -(2.0 ** 24), 1.0, 1.0
    b = np.zeros(K, np.float32)
    b[0], b[8], b[128], b[136] = 2.0 ** 24, -(2.0 ** 24), 1.0, 1.0
    return a, b


def _ln_by_hand(x, mu, var, eps=np.float32(0.0)):
    """y = ((x - mu) * rstd) * 1 + 0 from given moments, each step one fp32
    rounding (numpy float32 arithmetic is IEEE round-to-nearest)."""
    rstd = np.float32(1.0) / np.sqrt(np.float32(var) + eps)
    return ((x - np.float32(mu)) * rstd).astype(np.float32)


def test_layernorm_canonical_order_rows(orc):
    """The fixed LayerNorm reduction order (128 slots, xor-16-first butterfly,
    groups as (r0 + r2) + (r1 + r3)) on two hand-built rows whose fp32 mean
    is 2^-10 under that order and 2^-9 under the plausible others (see the
    comment above): y equals the hand-derived values bit for bit and differs
    from the alternative mean's."""
    g = np.ones(1024, np.float32)
    for x in _order_rows():
        y = orc.layernorm_row(x, g, None, eps=0.0)
        want = _ln_by_hand(x, 2.0 ** -10, 2.0 ** 39)
        assert np.array_equal(y.view(np.uint32), want.view(np.uint32))
        alt = _ln_by_hand(x, 2.0 ** -9, 2.0 ** 39)
        assert not np.array_equal(y, alt)


def test_quant_act_rms_exact_rows(orc):
    """The RMSNorm quantizer pinned by hand.  Rows of +-2 with eps = 0: the
    mean of squares is exactly 4 in any order, rstd = 1/2, so y = +-gamma'.
    Per token, the row peak 4 gives Delta = 4/127 and 1/Delta = 31.75 exactly,
    so gamma' = 4, 1, 0.5, 2, 3, 0.25, 1.5, 0.75 code to 127, 32, 16 (15.875),
    64 (63.5, tie to even), 95 (95.25), 8 (7.9375), 48 (47.625), 24 (23.8125).
    Static step 1/32: 4 -> 128 saturates to 127 (counted), the others to 32,
    16, 64, 96, 8, 48, 24.  Per-tensor dynamic over both rows: peak 4 again,
    so the per-token codes.  The rows' mean is 1, not 0: a LayerNorm in place
    of the RMSNorm would shift and rescale y and change the codes."""
    gp = np.array([4, 1, 0.5, 2, 3, 0.25, 1.5, 0.75] * 2, np.float32)
    sign = np.array([[1, -1, 1, 1, -1, 1, 1, 1, 1, -1, 1, 1, 1, 1, -1, 1],
                     [-1, 1, 1, 1, 1, -1, 1, 1, 1, 1, -1, 1, 1, 1, 1, -1]], np.float32)
    x = (2.0 * sign).astype(np.float32)
    mag_tok = np.array([127, 32, 16, 64, 95, 8, 48, 24] * 2)
    mag_st = np.array([127, 32, 16, 64, 96, 8, 48, 24] * 2)
    xq, act, ncl = orc.quant_act_rms(x, gp, eps=0.0, per_token=True)
    assert np.array_equal(act, np.full(2, np.float32(4.0) / np.float32(127.0)))
    assert np.array_equal(xq, (sign * mag_tok).astype(np.int8)) and ncl == 0
    xq, _, ncl = orc.quant_act_rms(x, gp, eps=0.0, per_token=False,
                                   static_delta=np.float32(1.0 / 32))
    assert np.array_equal(xq, (sign * mag_st).astype(np.int8)) and ncl == 4
    xq, act, _ = orc.quant_act_rms(x, gp, eps=0.0, per_tensor_dynamic=True)
    assert act[0] == np.float32(4.0) / np.float32(127.0)
    assert np.array_equal(xq, (sign * mag_tok).astype(np.int8))
    xq_ln, _, _ = orc.quant_act(x, gp, None, 0.0, per_token=True)
    assert not np.array_equal(xq_ln, (sign * mag_tok).astype(np.int8))


def test_quant_act_rms_through_rmsnorm_row(orc):
    """The RMSNorm quantizer equals the separately pinned RMSNorm row
    (orc.rmsnorm_row) followed by the textbook quantizer written out here in
    fp32 numpy -- Delta = max(peak, 1e-7)/127, codes rne(y * (1/Delta))
    clamped to +-127 -- on outlier-structured rows, per token, static and per
    tensor dynamic."""
    lin = synth.workloads()["tiny_k1024"].linears[0]
    d = synth.make_linear_inputs(lin, T=12, T_cal=16, N=8)
    g = (1 + 0.1 * np.random.default_rng(15).standard_normal(1024)).astype(np.float32)
    y = np.stack([orc.rmsnorm_row(row, g) for row in d["x"]])

    def q(yv, dl):
        inv = np.float32(1.0) / np.float32(dl)
        return np.clip(np.rint(yv * inv), -127, 127).astype(np.int8)

    def dlt(peak):
        return np.float32(max(np.float32(peak), np.float32(1e-7))) / np.float32(127.0)

    xq, act, _ = orc.quant_act_rms(d["x"], g, per_token=True)
    for t in range(y.shape[0]):
        assert act[t] == dlt(np.abs(y[t]).max())
        assert np.array_equal(xq[t], q(y[t], act[t]))
    ds = np.float32(0.02)
    xq, _, ncl = orc.quant_act_rms(d["x"], g, per_token=False, static_delta=ds)
    assert np.array_equal(xq, q(y, ds))
    assert ncl == int(np.sum(np.abs(np.rint(y * (np.float32(1) / ds))) > 127))
    xq, act, _ = orc.quant_act_rms(d["x"], g, per_tensor_dynamic=True)
    assert act[0] == dlt(np.abs(y).max())
    assert np.array_equal(xq, q(y, act[0]))


def test_rmsnorm_fold_alpha_one(orc):
    """Calibration through the RMSNorm, alpha = 1 (s = the peaks), the fold
    gamma' = gamma / s: the smoothed calibration peaks are 1 within 2 ulp
    (y' = ((x * rstd) * gamma) / s against (x * rstd) * (gamma / s)), and the
    quantizer's per-token path equals its per-tensor-dynamic path on one row."""
    lin = synth.workloads()["tiny_k1024"].linears[0]
    d = synth.make_linear_inputs(lin, T=16, T_cal=64, N=8)
    g = (1 + 0.1 * np.random.default_rng(14).standard_normal(1024)).astype(np.float32)
    amax = orc.calib_absmax_rms(d["x_cal"], g)
    s, _ = orc.smooth_scales(amax, np.ones(1024, np.float32), 1.0)
    assert np.array_equal(s, np.maximum(amax, np.float32(1e-4)))
    g2 = (g / s).astype(np.float32)
    peak = orc.calib_absmax_rms(d["x_cal"], g2)
    assert max(ulps(p, 1.0) for p in peak) <= 2
    xq1, a1, _ = orc.quant_act_rms(d["x"][3:4], g2, per_token=True)
    xq2, a2, _ = orc.quant_act_rms(d["x"][3:4], g2, per_tensor_dynamic=True)
    assert a1[0] == a2[0] and np.array_equal(xq1, xq2)


def test_fold_into_producer(orc):
    """Folding 1/s into the producing linear ([review] §5.5): with
    power-of-two s the divisions are exact; on general data the producer's
    output with the folded scale and bias equals its original output divided
    by s within 2 ulp (fp64 reference), a ReLU in between commutes (s > 0),
    and the consumer then needs no 1/s: quantizing the folded output with
    inv_s NULL equals quantizing the original output times 1/s on all but
    last-bit ties."""
    r = np.random.default_rng(31)
    K = 64
    s2 = (2.0 ** r.integers(-6, 7, K)).astype(np.float32)
    ws = r.uniform(1e-4, 1e-2, K).astype(np.float32)
    b = r.normal(0, 0.5, K).astype(np.float32)
    ws2, b2 = orc.fold_into_producer(s2, ws, b)
    assert np.array_equal(ws2, ws / s2) and np.array_equal(b2, b / s2)
    # producer: M x Kp -> K outputs (its output channels = consumer inputs)
    M, Kp = 24, 96
    xq = r.integers(-127, 128, (M, Kp)).astype(np.int8)
    wq = r.integers(-127, 128, (K, Kp)).astype(np.int8)
    act = r.uniform(1e-3, 1e-1, M).astype(np.float32)
    s = r.uniform(0.05, 20.0, K).astype(np.float32)
    y, acc = orc.gemm_w8a8(xq, wq, act, ws, bias=b)
    wsf, bf = orc.fold_into_producer(s, ws, b)
    yf, acc_f = orc.gemm_w8a8(xq, wq, act, wsf, bias=bf)
    assert np.array_equal(acc, acc_f)
    term = acc.astype(np.float64) * act[:, None] * ws[None, :] / s[None, :]
    ref = term + b[None, :] / s[None, :]
    # four fp32 roundings, each relative to the terms (a sum may cancel)
    bound = 4 * F32_EPS * (np.abs(term) + np.abs(b / s)[None, :])
    assert np.all(np.abs(yf - ref) <= bound)
    assert np.array_equal(np.maximum(yf, 0) > 0, np.maximum(ref, 0) > 0)
    xq_f, a_f, _ = orc.quant_act(np.maximum(yf, 0).astype(np.float32), per_token=True)
    xq_o, a_o, _ = orc.quant_act(np.maximum(y, 0).astype(np.float32),
                                 inv_s=(1.0 / s).astype(np.float32), per_token=True)
    assert np.mean(xq_f == xq_o) > 0.99 and np.max(np.abs(xq_f.astype(int) - xq_o)) <= 1


def test_output_error_closed_forms(orc):
    """The layer-output error metric: 0 for y = y_ref, 1 for y = 2 y_ref or
    y = 0, and scale-invariant."""
    r = np.random.default_rng(41).normal(0, 3, (7, 5)).astype(np.float32)
    assert orc.output_error(r, r) == 0.0
    assert orc.output_error(2 * r, r) == pytest.approx(1.0, rel=1e-15)
    assert orc.output_error(np.zeros_like(r), r) == 1.0
    assert orc.output_error(8 * r + 8, 8 * r) == pytest.approx(orc.output_error(r + 1, r),
                                                                rel=1e-12)


def test_alpha_sweep_u_shape(orc):
    """Layer-output error against alpha on outlier-structured data ([review]
    §5.3 eq. (4) and its alpha discussion: alpha = 0 leaves the activation
    outliers in X, alpha = 1 moves them all into W; the paper's sweep, Fig. 10,
    has its sweet spot in between).  Reference: the unquantized layer in
    fp64.  The error at 0.5 is below both ends, for per-token and static
    activations, with and without a LayerNorm."""
    lin = synth.workloads()["tiny_k1024"].linears[0]
    d = synth.make_linear_inputs(lin, T=64, T_cal=256, N=256)
    x, x_cal, w = d["x"], d["x_cal"], d["w"]
    for ln in (False, True):
        g, b = (d["gamma"], d["beta"]) if ln else (None, None)
        amax = orc.calib_absmax(x_cal, g, b)
        f = (orc.layernorm_row(x[t], g, b) for t in range(x.shape[0])) if ln else iter(x)
        fx = np.stack(list(f)).astype(np.float64)
        y_ref = (fx @ w.astype(np.float64).T).astype(np.float32)
        for gran in ("token", "static"):
            e = {a: orc.alpha_error(amax, w, x, y_ref, a, g, b, gran=gran) for a in (0.0, 0.5, 1.0)}
            assert e[0.5] < e[0.0] and e[0.5] < e[1.0], (ln, gran, e)


def test_calib_absmax_running_and_library(orc):
    """S1 raw mode equals numpy's max(|X|) over tokens, and a running max
    over two batches equals the max over their concatenation."""
    lin = synth.workloads()["opt6.7b_qkv_t2048"].linears[0]
    d = synth.make_linear_inputs(lin, T=8, T_cal=40, N=8)
    xf = synth.bf16_bits_to_f32(d["x_cal"])
    a = orc.calib_absmax(d["x_cal"])
    assert np.array_equal(a, np.abs(xf).max(axis=0))
    a1 = orc.calib_absmax(d["x_cal"][:17])
    a2 = orc.calib_absmax(d["x_cal"][17:], amax=a1)
    assert np.array_equal(a2, a)
    # LN mode: the statistic of each LN row
    aln = orc.calib_absmax(d["x_cal"], d["gamma"], d["beta"])
    ref = np.zeros_like(aln)
    for t in range(40):
        ref = np.maximum(ref, np.abs(orc.layernorm_row(xf[t], d["gamma"], d["beta"])))
    assert np.array_equal(aln, ref)


def test_weight_colmax_library(orc):
    r = np.random.default_rng(11)
    w = r.standard_normal((33, 48)).astype(np.float32)
    assert np.array_equal(orc.weight_colmax(w), np.abs(w).max(axis=0))
    wb = synth.bf16_bits(w)
    assert np.array_equal(orc.weight_colmax(wb), np.abs(synth.bf16_bits_to_f32(wb)).max(axis=0))


def test_fuse_weights_properties(orc):
    """Per-output-channel symmetric INT8 of W*s: each row's peak hits +-127
    and every code is within half a step of W*s."""
    r = np.random.default_rng(12)
    w = (r.standard_normal((20, 64)) * 0.02).astype(np.float32)
    s = r.uniform(0.1, 20, 64).astype(np.float32)
    wq, ws = orc.fuse_weights_q8(w, s)
    wh = w * s[None, :]
    for n in range(20):
        assert ws[n] == orc.delta(float(np.abs(wh[n]).max()))
        assert np.abs(wq[n]).max() == 127
        err = np.abs(wh[n].astype(np.float64) - np.float64(ws[n]) * wq[n])
        assert np.all(err <= ws[n] / 2 * (1 + 1e-5))


def test_fold_ln_is_division(orc):
    """gamma' = gamma/s and beta' = beta/s ([embedded] §二): multiplying back
    recovers gamma and beta to within one rounding."""
    r = np.random.default_rng(13)
    g = r.uniform(0.5, 1.5, 64).astype(np.float32)
    b = r.uniform(-0.1, 0.1, 64).astype(np.float32)
    s = r.uniform(0.01, 50, 64).astype(np.float32)
    g2, b2 = orc.fold_ln(g, b, s)
    assert np.all(np.abs(g2.astype(np.float64) * s - g) <= np.abs(g) * 2 * F32_EPS)
    assert np.all(np.abs(b2.astype(np.float64) * s - b) <= np.abs(b) * 2 * F32_EPS)


# ------------------------------------------------------------------ P-9

def test_smoothing_raises_effective_levels(orc):
    """[review] §2.4: a channel with peak m_i in a tensor with peak m gets
    about 2^8 m_i/m effective levels; smoothing (alpha 0.5) raises them for
    the ordinary channels of the outlier-structured workload."""
    lin = synth.workloads()["tiny_k1024"].linears[0]
    d = synth.make_linear_inputs(lin, T=8, T_cal=512, N=256)
    amax = orc.calib_absmax(d["x_cal"])
    s, _ = orc.smooth_scales(amax, orc.weight_colmax(d["w"]), 0.5)
    before = 256 * amax / amax.max()
    sm = amax / s
    after = 256 * sm / sm.max()
    ordinary = np.setdiff1d(np.arange(1024), d["outliers"].channels)
    assert np.median(after[ordinary]) > 4 * np.median(before[ordinary])
