"""GPU parity of the HBM-bound steps against the CPU oracle, element by
element on the same seeded inputs (bit-exact: peaks, scales, codes).

Shapes span several slices/strips plus ragged tails, both element types, and
the register-cached and re-reading row variants."""
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


def _x(seed, T, K, dtype, frac=0.01, relu=False):
    out = synth.outlier_pattern(seed, K, frac)
    x = synth.activations(seed, f"x{T}x{K}", T, K, out, relu=relu)
    return synth.bf16_bits(x) if dtype == "bf16" else x


def _ln(seed, K):
    return synth.ln_params(seed, f"ln{K}", K)


SHAPES_RAW = [(1, 16), (37, 48), (300, 1040), (1000, 4096), (77, 12288)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,K", SHAPES_RAW)
def test_calib_absmax_raw(sq, orc, dtype, T, K):
    x = _x(7, T, K, dtype)
    want = orc.calib_absmax(x)
    amax = torch.zeros(K, dtype=torch.float32, device="cuda")
    sq.sq_calib_absmax(dev(x), amax)
    assert_bits_equal(host(amax), want, "amax")
    # running maximum across a second batch
    x2 = _x(8, max(1, T // 2), K, dtype)
    sq.sq_calib_absmax(dev(x2), amax)
    assert_bits_equal(host(amax), orc.calib_absmax(x2, amax=want), "amax running")


SHAPES_LN = [(1, 16), (5, 48), (33, 1040), (130, 4096), (64, 5120), (9, 8192), (12, 12288),
             (3, 20480), (2, 53248)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,K", SHAPES_LN)
def test_calib_absmax_layernorm(sq, orc, dtype, T, K):
    x = _x(9, T, K, dtype)
    g, b = _ln(9, K)
    want = orc.calib_absmax(x, g, b, 1e-5)
    amax = torch.zeros(K, dtype=torch.float32, device="cuda")
    sq.sq_calib_absmax(dev(x), amax, dev(g), dev(b), 1e-5)
    assert_bits_equal(host(amax), want, "amax(LN)")
    # beta omitted
    want2 = orc.calib_absmax(x, g, None, 1e-5)
    amax.zero_()
    sq.sq_calib_absmax(dev(x), amax, dev(g), None, 1e-5)
    assert_bits_equal(host(amax), want2, "amax(LN, no beta)")


@pytest.mark.parametrize("alpha", [0.5, 0.0, 1.0, 0.8, 0.25])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,K", [(1, 16), (300, 1040), (777, 4096)])
def test_smooth_scales(sq, orc, alpha, dtype, N, K):
    r = np.random.default_rng(N + K)
    w = (r.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[:, 3] = 0.0  # an all-zero weight column: the 1e-7 floor
    if dtype == "bf16":
        w = synth.bf16_bits(w)
    amax = np.abs(_x(11, 64, K, "f32")).max(axis=0).astype(np.float32)
    amax[5] = 0.0  # a dead activation channel: the 1e-4 floor on s
    s_want, inv_want = orc.smooth_scales(amax, orc.weight_colmax(w), alpha)
    s = torch.empty(K, dtype=torch.float32, device="cuda")
    inv = torch.empty_like(s)
    dA = torch.empty(1, dtype=torch.float32, device="cuda")
    sq.sq_smooth_scales(dev(amax), dev(w), alpha, s, inv, dA)
    s_got, inv_got = host(s), host(inv)
    if alpha in (0.0, 0.5, 1.0):
        assert_bits_equal(s_got, s_want, "s")
        assert_bits_equal(inv_got, inv_want, "inv_s")
    else:
        # fp64 pow is not correctly rounded on either side: within 1 fp32 ulp
        assert ulp_diff_f32(s_got, s_want).max() <= 1
        assert_bits_equal(inv_got, (np.float32(1) / s_got).astype(np.float32), "inv_s")
    # the static step, recomputed by the oracle from the GPU's s
    assert_bits_equal(host(dA), np.array([orc.static_delta(amax, s_got)], np.float32), "delta_A")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,K", [(1, 16), (3, 48), (129, 1040), (300, 4096), (17, 20480),
                                 (5, 26624)])
def test_fuse_weights_q8(sq, orc, dtype, N, K):
    r = np.random.default_rng(N * K)
    w = (r.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[0, :] = 0.0  # an all-zero output channel
    if dtype == "bf16":
        w = synth.bf16_bits(w)
    s = r.uniform(0.05, 40.0, K).astype(np.float32)
    g = r.uniform(0.5, 1.5, K).astype(np.float32)
    b = r.uniform(-0.1, 0.1, K).astype(np.float32)
    wq_want, ws_want = orc.fuse_weights_q8(w, s)
    g_want, b_want = orc.fold_ln(g, b, s)
    wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    ws = torch.empty(N, dtype=torch.float32, device="cuda")
    g2 = torch.empty(K, dtype=torch.float32, device="cuda")
    b2 = torch.empty_like(g2)
    sq.sq_fuse_weights_q8(dev(w), dev(s), wq, ws, dev(g), dev(b), g2, b2)
    assert_bits_equal(host(ws), ws_want, "w_scale")
    assert_bits_equal(host(wq), wq_want, "wq")
    assert_bits_equal(host(g2), g_want, "gamma/s")
    assert_bits_equal(host(b2), b_want, "beta/s")


QUANT_SHAPES = [(1, 16), (3, 48), (37, 1040), (130, 4096), (9, 5120), (5, 12288), (4, 20480),
                (3, 26624)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", ["ln", "inv_s", "plain"])
@pytest.mark.parametrize("per_token", [True, False])
@pytest.mark.parametrize("T,K", QUANT_SHAPES)
def test_quant_act(sq, orc, dtype, mode, per_token, T, K):
    x = _x(13, T, K, dtype, relu=(mode == "plain"))
    r = np.random.default_rng(T + K)
    g = b = inv = None
    if mode == "ln":
        g, b = _ln(13, K)
        g = (g / r.uniform(0.5, 30, K)).astype(np.float32)  # folded gamma/s
    elif mode == "inv_s":
        inv = r.uniform(0.02, 2.0, K).astype(np.float32)
    dstatic = np.float32(0.05)  # small enough that the outliers saturate
    xq_want, act_want, ncl_want = orc.quant_act(
        x, g, b, 1e-5, inv, per_token=per_token, static_delta=dstatic)
    xq = torch.empty((T, K), dtype=torch.int8, device="cuda")
    act = (torch.empty(T, dtype=torch.float32, device="cuda") if per_token
           else torch.tensor([dstatic], dtype=torch.float32, device="cuda"))
    ncl = torch.zeros(1, dtype=torch.int64, device="cuda")
    sq.sq_ln_smooth_quant_act(dev(x), xq, act, dev(g), dev(b), 1e-5, dev(inv),
                              per_token=per_token, n_clipped=ncl)
    if per_token:
        assert_bits_equal(host(act), act_want, "act_scale")
    assert_bits_equal(host(xq), xq_want, "xq")
    assert int(host(ncl)[0]) == ncl_want


# The static step on bf16 rows without a norm runs whole rows held in
# registers: 512 threads of one chunk (K <= 4096) or two (K <= 8192), two rows
# a step, or 640 threads of four chunks (K <= 20480); wider rows take the
# column strips.  Each width at and just past its boundary, with row counts
# below, at and past the grid, odd (a last step of one row), and with
# saturating outliers counted.
ROWREG_STATIC = [(1, 4096), (149, 4096), (150, 4112), (297, 8192), (147, 8208),
                 (300, 20480), (5, 20496)]


@pytest.mark.parametrize("mode", ["inv_s", "plain"])
@pytest.mark.parametrize("T,K", ROWREG_STATIC)
def test_quant_act_static_rows_in_registers(sq, orc, mode, T, K):
    x = _x(41, T, K, "bf16", relu=(mode == "plain"))
    r = np.random.default_rng(T * 7 + K)
    inv = r.uniform(0.02, 2.0, K).astype(np.float32) if mode == "inv_s" else None
    dstatic = np.float32(0.04)
    xq_want, _, ncl_want = orc.quant_act(x, None, None, 1e-5, inv, per_token=False,
                                         static_delta=dstatic)
    xq = torch.empty((T, K), dtype=torch.int8, device="cuda")
    act = torch.tensor([dstatic], dtype=torch.float32, device="cuda")
    ncl = torch.zeros(1, dtype=torch.int64, device="cuda")
    sq.sq_ln_smooth_quant_act(dev(x), xq, act, None, None, 1e-5, dev(inv), per_token=False,
                              n_clipped=ncl)
    sq.sq_sync_status()
    assert_bits_equal(host(xq), xq_want, "xq")
    assert int(host(ncl)[0]) == ncl_want
    assert ncl_want > 0  # the outliers saturate


def test_quant_act_edge_values(sq, orc):
    """All-zero rows, +-inf and exact ties at the rounding boundary."""
    K = 64
    x = np.zeros((4, K), np.float32)
    x[1, :8] = [np.inf, -np.inf, 1.0, -1.0, 0.5, 2.5, -2.5, 3.0]
    x[2, :] = np.arange(K, dtype=np.float32) - 31.5
    x[3, :] = 1e-30
    for per_token in (True, False):
        d = np.float32(0.5)
        xq_want, act_want, ncl_want = orc.quant_act(x, per_token=per_token, static_delta=d)
        xq = torch.empty((4, K), dtype=torch.int8, device="cuda")
        act = (torch.empty(4, dtype=torch.float32, device="cuda") if per_token
               else torch.tensor([d], device="cuda"))
        ncl = torch.zeros(1, dtype=torch.int64, device="cuda")
        sq.sq_ln_smooth_quant_act(dev(x), xq, act, per_token=per_token, n_clipped=ncl)
        assert_bits_equal(host(xq), xq_want, "xq edge")
        if per_token:
            assert_bits_equal(host(act), act_want, "act edge")
        assert int(host(ncl)[0]) == ncl_want


def _with_non_finite(x, seed):
    """Rows with NaN among finite values (row 0: one NaN; row 1: several
    NaN and a +inf; row 2: all NaN; row 3: NaN beside the row's largest
    element), the rest of the rows untouched."""
    x = np.array(x, copy=True)
    r = np.random.default_rng(seed)
    K = x.shape[1]
    nan = np.float32(np.nan) if x.dtype == np.float32 else synth.bf16_bits(np.float32(np.nan))[0]
    inf = np.float32(np.inf) if x.dtype == np.float32 else synth.bf16_bits(np.float32(np.inf))[0]
    x[0, r.integers(0, K)] = nan
    x[1, r.integers(0, K, 5)] = nan
    x[1, r.integers(0, K)] = inf
    x[2, :] = nan
    mag = np.abs(x[3].astype(np.float32)) if x.dtype == np.float32 else np.abs(
        (x[3].astype(np.uint32) << 16).view(np.float32))
    k = int(np.argmax(mag))
    x[3, (k + 1) % K] = nan
    return x


NAN_SHAPES = [(6, 64), (5, 1040), (7, 4096), (4, 20480)]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", ["ln", "inv_s", "plain"])
@pytest.mark.parametrize("gran", ["token", "static", "tensor"])
@pytest.mark.parametrize("T,K", NAN_SHAPES)
def test_quant_act_nan_rows(sq, orc, dtype, mode, gran, T, K):
    """NaN (and +inf) in per-token, static and per-tensor-dynamic rows, with
    a LayerNorm, a 1/s multiplier or neither: NaN codes to 0, the peaks skip
    NaN, a LayerNorm row with a NaN is NaN throughout (all codes 0, the
    floored step); codes, steps and saturation counts bit-exact."""
    x = _with_non_finite(_x(41, T, K, dtype), T * K)
    r = np.random.default_rng(K)
    g = b = inv = None
    if mode == "ln":
        g, b = _ln(41, K)
    elif mode == "inv_s":
        inv = r.uniform(0.02, 2.0, K).astype(np.float32)
    dstatic = np.float32(0.05)
    kw = dict(per_token=(gran == "token"), static_delta=dstatic,
              per_tensor_dynamic=(gran == "tensor"))
    xq_want, act_want, ncl_want = orc.quant_act(x, g, b, 1e-5, inv, **kw)
    xq = torch.empty((T, K), dtype=torch.int8, device="cuda")
    if gran == "token":
        act = torch.empty(T, dtype=torch.float32, device="cuda")
    else:
        act = torch.tensor([dstatic], dtype=torch.float32, device="cuda")
    ncl = torch.zeros(1, dtype=torch.int64, device="cuda")
    sq.sq_ln_smooth_quant_act(dev(x), xq, act, dev(g), dev(b), 1e-5, dev(inv),
                              per_token=(gran == "token"), n_clipped=ncl,
                              per_tensor_dynamic=(gran == "tensor"))
    sq.sq_sync_status()
    if gran != "static":
        assert_bits_equal(host(act), act_want, "act_scale (NaN rows)")
    assert_bits_equal(host(xq), xq_want, "xq (NaN rows)")
    assert int(host(ncl)[0]) == ncl_want


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("ln", [False, True])
@pytest.mark.parametrize("T,K", [(40, 1040), (9, 4096), (300, 8192)])
def test_calib_absmax_nan_rows(sq, orc, dtype, ln, T, K):
    """Calibration peaks skip NaN (raw column strips and LayerNorm rows)."""
    x = _with_non_finite(_x(43, T, K, dtype), T + K)
    g, b = _ln(43, K) if ln else (None, None)
    want = orc.calib_absmax(x, g, b, 1e-5)
    amax = torch.zeros(K, dtype=torch.float32, device="cuda")
    sq.sq_calib_absmax(dev(x), amax, dev(g), dev(b), 1e-5)
    assert_bits_equal(host(amax), want, "amax (NaN rows)")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_layernorm_order_rows(sq, orc, dtype):
    """The two hand-built rows whose fp32 mean depends on the canonical
    LayerNorm reduction order (the oracle is pinned on them by hand), with
    seeded rows beside them: calibration peak and per-token / static codes
    bit-exact against the oracle, eps = 0 and 1e-5."""
    K = 1024
    ra = np.zeros(K, np.float32)
    ra[0], ra[256], ra[512], ra[768] = 2.0 ** 24, -(2.0 ** 24), 1.0, 1.0
    rb = np.zeros(K, np.float32)
    rb[0], rb[8], rb[128], rb[136] = 2.0 ** 24, -(2.0 ** 24), 1.0, 1.0
    x = np.concatenate([ra[None], rb[None], _x(45, 6, K, "f32")]).astype(np.float32)
    if dtype == "bf16":
        x = synth.bf16_bits(x)
    g = np.ones(K, np.float32)
    gs, bs = _ln(45, K)
    for eps in (0.0, 1e-5):
        for gg, bb in ((g, None), (gs, bs)):
            want = orc.calib_absmax(x, gg, bb, eps)
            amax = torch.zeros(K, dtype=torch.float32, device="cuda")
            sq.sq_calib_absmax(dev(x), amax, dev(gg), dev(bb), eps)
            assert_bits_equal(host(amax), want, "amax (order rows)")
            for per_token in (True, False):
                dstatic = np.float32(1e-4)
                xq_want, act_want, _ = orc.quant_act(x, gg, bb, eps, per_token=per_token,
                                                     static_delta=dstatic)
                xq = torch.empty((x.shape[0], K), dtype=torch.int8, device="cuda")
                act = (torch.empty(x.shape[0], dtype=torch.float32, device="cuda") if per_token
                       else torch.tensor([dstatic], device="cuda"))
                sq.sq_ln_smooth_quant_act(dev(x), xq, act, dev(gg), dev(bb), eps,
                                          per_token=per_token)
                if per_token:
                    assert_bits_equal(host(act), act_want, "act (order rows)")
                assert_bits_equal(host(xq), xq_want, "xq (order rows)")


def test_runs_are_deterministic(sq):
    """Two runs of the LN calibration and the quantizer give identical bits
    (a race in the reductions would show up here)."""
    K, T = 4096, 257
    x = dev(_x(21, T, K, "bf16"))
    g, b = _ln(21, K)
    g, b = dev(g), dev(b)
    outs = []
    for _ in range(2):
        amax = torch.zeros(K, dtype=torch.float32, device="cuda")
        sq.sq_calib_absmax(x, amax, g, b)
        xq = torch.empty((T, K), dtype=torch.int8, device="cuda")
        act = torch.empty(T, dtype=torch.float32, device="cuda")
        sq.sq_ln_smooth_quant_act(x, xq, act, g, b)
        outs.append((host(amax), host(xq), host(act)))
    for a, b_ in zip(outs[0], outs[1]):
        assert_bits_equal(a, b_, "rerun")


# Enough rows that every CTA of the row pipeline cycles its shared-memory
# ring several times (rows per CTA > ring slots), for each ring geometry:
# 16 slots / 8 slices, 8 / 8, 4 / 4 and 2 slots shared by two 8-warp slices.
RING_CASES = [
    (5000, 4096, "ln", True), (2500, 5120, "ln", True), (2500, 8192, "inv_s", False),
    (1300, 12288, "inv_s", True), (700, 20480, "plain", True), (700, 20480, "inv_s", False),
]


@pytest.mark.parametrize("T,K,mode,per_token", RING_CASES)
def test_quant_act_ring_reuse(sq, orc, T, K, mode, per_token):
    x = _x(31, T, K, "bf16", relu=(mode == "plain"))
    r = np.random.default_rng(T * K)
    g = b = inv = None
    if mode == "ln":
        g, b = _ln(31, K)
    elif mode == "inv_s":
        inv = r.uniform(0.02, 2.0, K).astype(np.float32)
    dstatic = np.float32(0.05)
    xq_want, act_want, ncl_want = orc.quant_act(
        x, g, b, 1e-5, inv, per_token=per_token, static_delta=dstatic)
    xq = torch.empty((T, K), dtype=torch.int8, device="cuda")
    act = (torch.empty(T, dtype=torch.float32, device="cuda") if per_token
           else torch.tensor([dstatic], dtype=torch.float32, device="cuda"))
    ncl = torch.zeros(1, dtype=torch.int64, device="cuda")
    sq.sq_ln_smooth_quant_act(dev(x), xq, act, dev(g), dev(b), 1e-5, dev(inv),
                              per_token=per_token, n_clipped=ncl)
    sq.sq_sync_status()
    if per_token:
        assert_bits_equal(host(act), act_want, "act_scale")
    assert_bits_equal(host(xq), xq_want, "xq")
    assert int(host(ncl)[0]) == ncl_want


@pytest.mark.parametrize("T,K", [(3000, 4096), (3000, 5120), (2000, 1024)])
def test_calib_absmax_layernorm_ring_reuse(sq, orc, T, K):
    x = _x(33, T, K, "bf16")
    g, b = _ln(33, K)
    want = orc.calib_absmax(x, g, b, 1e-5)
    amax = torch.zeros(K, dtype=torch.float32, device="cuda")
    sq.sq_calib_absmax(dev(x), amax, dev(g), dev(b), 1e-5)
    sq.sq_sync_status()
    assert_bits_equal(host(amax), want, "amax(LN)")


@pytest.mark.parametrize("N,K", [(700, 20480), (1300, 12288), (5000, 4096)])
def test_fuse_weights_ring_reuse(sq, orc, N, K):
    r = np.random.default_rng(N + K)
    w = synth.bf16_bits((r.standard_normal((N, K)) * 0.02).astype(np.float32))
    s = r.uniform(0.05, 40.0, K).astype(np.float32)
    wq_want, ws_want = orc.fuse_weights_q8(w, s)
    wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    ws = torch.empty(N, dtype=torch.float32, device="cuda")
    sq.sq_fuse_weights_q8(dev(w), dev(s), wq, ws)
    sq.sq_sync_status()
    assert_bits_equal(host(ws), ws_want, "w_scale")
    assert_bits_equal(host(wq), wq_want, "wq")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N,K", [(1, 16), (300, 1040), (12288, 4096), (77, 20480)])
@pytest.mark.parametrize("alpha", [0.5, 0.8, 0.0, 1.0])
def test_weight_peaks_then_scales(sq, orc, dtype, N, K, alpha):
    """sq_weight_colmax + sq_smooth_scales_peaks (the weight peaks computed on
    their own, e.g. concurrently with the calibration) give the weight peaks
    of the oracle and the same bits as the one-call sq_smooth_scales,
    including the static step."""
    w = _x(N + K, N, K, dtype)
    amax_x = np.abs(_x(K, 64, K, "f32")).max(axis=0).astype(np.float32)
    f32 = dict(dtype=torch.float32, device="cuda")
    amax_w = torch.empty(K, **f32)
    sq.sq_weight_colmax(dev(w), amax_w)
    s1, i1, d1 = torch.empty(K, **f32), torch.empty(K, **f32), torch.empty(1, **f32)
    sq.sq_smooth_scales_peaks(dev(amax_x), amax_w, alpha, s1, i1, d1)
    s2, i2, d2 = torch.empty(K, **f32), torch.empty(K, **f32), torch.empty(1, **f32)
    sq.sq_smooth_scales(dev(amax_x), dev(w), alpha, s2, i2, d2)
    sq.sq_sync_status()
    assert_bits_equal(host(amax_w), orc.weight_colmax(w), "amax_w")
    for a, b, what in ((s1, s2, "s"), (i1, i2, "inv_s"), (d1, d2, "delta_A")):
        assert_bits_equal(host(a), host(b), what)
