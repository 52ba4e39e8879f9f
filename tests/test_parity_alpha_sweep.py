"""GPU parity of the alpha sweep (NEXT-2: alpha chosen by the layer's output
error, [review] §5.3): the whole smoothed W8A8 layer runs on the GPU for
each alpha and its relative Frobenius error against a reference output is
compared with the oracle's same chain.  The layer outputs are bit-exact for
alpha in {0, 0.5, 1}, so the errors agree to the fp64 summation order; for
other alpha the factors may differ by one fp32 ulp (neither fp64 pow is
correctly rounded), so the errors agree to 1e-3 relative."""
import dataclasses

import numpy as np
import pytest

import synth
from tests._util import dev, host

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import w8a8_int8_gemm_calib_b200 as m

    return m


def _case(dtype, ln, T=64, T_cal=256, N=256, K=None):
    lin = synth.workloads()["tiny_k1024"].linears[0]
    if K is not None:
        lin = dataclasses.replace(lin, K=K)
    d = synth.make_linear_inputs(lin, T=T, T_cal=T_cal, N=N)
    x, x_cal, w = d["x"], d["x_cal"], d["w"]
    if dtype == "bf16":
        x, x_cal, w = synth.bf16_bits(x), synth.bf16_bits(x_cal), synth.bf16_bits(w)
    g, b = (d["gamma"], d["beta"]) if ln else (None, None)
    return x, x_cal, w, g, b


def _ref(orc, x, w, g, b):
    xf = synth.bf16_bits_to_f32(x) if x.dtype == np.uint16 else x
    wf = synth.bf16_bits_to_f32(w) if w.dtype == np.uint16 else w
    if g is not None:
        xf = np.stack([orc.layernorm_row(r, g, b) for r in xf])
    return (xf.astype(np.float64) @ wf.astype(np.float64).T).astype(np.float32)


ALPHAS = [0.0, 0.25, 0.5, 0.75, 1.0]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("ln", [False, True])
@pytest.mark.parametrize("gran", ["token", "static", "tensor"])
def test_alpha_sweep(sq, orc, dtype, ln, gran):
    x, x_cal, w, g, b = _case(dtype, ln)
    amax = orc.calib_absmax(x_cal, g, b)
    y_ref = _ref(orc, x, w, g, b)
    want = [orc.alpha_error(amax, w, x, y_ref, a, g, b, gran=gran) for a in ALPHAS]
    err = sq.sq_alpha_sweep(dev(amax), dev(w), dev(x), dev(y_ref), ALPHAS, dev(g), dev(b),
                            per_token=gran == "token", per_tensor_dynamic=gran == "tensor")
    sq.sq_sync_status()
    got = host(err)
    for a, e_got, e_want in zip(ALPHAS, got, want):
        tol = 1e-9 if a in (0.0, 0.5, 1.0) else 1e-3
        assert abs(e_got - e_want) <= tol * e_want, (a, e_got, e_want)
    # the sweet spot lies inside
    assert got[2] < got[0] and got[2] < got[4]


def test_alpha_sweep_larger_bf16_layer(sq, orc):
    """A 512 x 2048 x 1024 bf16 layer with a LayerNorm, per-token: errors
    against the oracle and the U-shape."""
    x, x_cal, w, g, b = _case("bf16", True, T=512, T_cal=512, N=2048)
    amax = orc.calib_absmax(x_cal, g, b)
    y_ref = _ref(orc, x, w, g, b)
    alphas = [0.0, 0.5, 1.0]
    want = [orc.alpha_error(amax, w, x, y_ref, a, g, b) for a in alphas]
    ws = sq.Workspace()
    err = sq.sq_alpha_sweep(dev(amax), dev(w), dev(x), dev(y_ref), alphas, dev(g), dev(b),
                            workspace=ws)
    again = sq.sq_alpha_sweep(dev(amax), dev(w), dev(x), dev(y_ref), alphas[::-1], dev(g),
                              dev(b), workspace=ws)
    sq.sq_sync_status()
    got = host(err)
    for e_got, e_want in zip(got, want):
        assert abs(e_got - e_want) <= 1e-9 * e_want
    assert np.array_equal(host(again)[::-1], got)  # reuse, any order: deterministic sums
    assert got[1] < got[0] and got[1] < got[2]


@pytest.mark.parametrize("T,N,K", [(300, 264, 1024), (200, 520, 256)])
@pytest.mark.parametrize("gran,dtype,ln", [("token", "bf16", True), ("static", "f32", False),
                                           ("tensor", "bf16", False)])
def test_alpha_sweep_error_in_gemm_epilogue(sq, orc, T, N, K, gran, dtype, ln):
    """More than 128 tokens: the GEMM folds the error sums into its epilogue
    (one fp64 pair per each of its 12 epilogue warps) and never writes y.
    Ragged rows and columns, a long and a short K; errors against the
    oracle's same chain, and bit-identical on a second run."""
    x, x_cal, w, g, b = _case(dtype, ln, T=T, T_cal=256, N=N, K=K)
    amax = orc.calib_absmax(x_cal, g, b)
    y_ref = _ref(orc, x, w, g, b)
    alphas = [0.0, 0.5, 1.0]
    want = [orc.alpha_error(amax, w, x, y_ref, a, g, b, gran=gran) for a in alphas]
    kw = dict(per_token=gran == "token", per_tensor_dynamic=gran == "tensor")
    err = sq.sq_alpha_sweep(dev(amax), dev(w), dev(x), dev(y_ref), alphas, dev(g), dev(b), **kw)
    again = sq.sq_alpha_sweep(dev(amax), dev(w), dev(x), dev(y_ref), alphas, dev(g), dev(b), **kw)
    sq.sq_sync_status()
    got = host(err)
    for a, e_got, e_want in zip(alphas, got, want):
        assert abs(e_got - e_want) <= 1e-9 * e_want, (a, e_got, e_want)
    assert np.array_equal(host(again), got)
