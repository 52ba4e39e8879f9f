"""GPU parity of the batched INT8 GEMM (NEXT-4: the attention block's INT8
matmuls, [review] §5.6 Fig. 6) against the oracle's per-batch GEMM: INT32
accumulators and fp32 / bf16 outputs bit for bit.  Shapes cover attention
(scores Q K^T with a head dimension of 64 or 128, P V with V^T as the K-major
operand), ragged rows and columns inside each batch (the 3-D tensor maps zero-
fill and clip at every batch's own edge), a single token, and all four scale
combinations."""
import numpy as np
import pytest

from tests._util import assert_bits_equal, dev, host

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import w8a8_int8_gemm_calib_b200 as m

    return m


def _operands(B, M, N, K, per_token, per_channel, seed):
    r = np.random.default_rng(seed)
    xq = r.integers(-127, 128, (B, M, K)).astype(np.int8)
    wq = r.integers(-127, 128, (B, N, K)).astype(np.int8)
    act = r.uniform(1e-3, 0.1, B * M if per_token else B).astype(np.float32)
    ws = r.uniform(1e-4, 1e-2, B * N if per_channel else B).astype(np.float32)
    return xq, wq, act, ws


def _run(sq, xq, wq, act, ws, per_token, per_channel, out):
    B, M, _ = xq.shape
    N = wq.shape[1]
    y = torch.empty((B, M, N), dtype=torch.bfloat16 if out == "bf16" else torch.float32,
                    device="cuda")
    acc = torch.empty((B, M, N), dtype=torch.int32, device="cuda")
    sq.sq_bmm_w8a8(dev(xq), dev(wq), dev(act), dev(ws), y, per_token=per_token,
                   w_per_channel=per_channel, acc_out=acc)
    sq.sq_sync_status()
    return host(y), host(acc)


SHAPES = [(1, 128, 256, 128), (3, 17, 33, 64), (32, 256, 256, 128), (32, 256, 128, 256),
          (5, 129, 200, 48), (2, 1, 1000, 2064), (7, 300, 72, 64), (4, 64, 64, 4096)]


@pytest.mark.parametrize("B,M,N,K", SHAPES)
@pytest.mark.parametrize("out", ["f32", "bf16"])
@pytest.mark.parametrize("per_token,per_channel", [(True, True), (False, False),
                                                   (True, False), (False, True)])
def test_bmm(sq, orc, B, M, N, K, out, per_token, per_channel):
    xq, wq, act, ws = _operands(B, M, N, K, per_token, per_channel, B * 1000 + M + N + K)
    y_want, acc_want = orc.bmm_w8a8(xq, wq, act, ws, per_token, per_channel,
                                    out_bf16=(out == "bf16"))
    y, acc = _run(sq, xq, wq, act, ws, per_token, per_channel, out)
    assert_bits_equal(acc, acc_want, "acc")
    assert_bits_equal(y, y_want, "y")


@pytest.mark.parametrize("B,M,N,K", [(3, 130, 200, 240), (3, 130, 200, 256), (3, 130, 200, 272),
                                     (3, 130, 200, 512), (3, 130, 200, 528), (2, 1024, 2048, 64)])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_bmm_short_k_epilogue(sq, orc, B, M, N, K, out):
    """Head-sized K: three epilogue warps per accumulator quarter up to four
    k-blocks (K = 528 is back on one), with the largest accumulators the
    codes allow beside random rows (2^22 at K = 256).  130 x 200 per batch picks the
    128-column tile (four chunks over three warps), 1024 x 2048 the
    256-column one."""
    r = np.random.default_rng(K + M)
    xq = r.integers(-128, 128, (B, M, K)).astype(np.int8)
    wq = r.integers(-128, 128, (B, N, K)).astype(np.int8)
    xq[:, :2] = -128
    wq[:, :2] = -128
    wq[1, 5] = 127
    act = r.uniform(1e-3, 0.1, B * M).astype(np.float32)
    ws = r.uniform(1e-4, 1e-2, B).astype(np.float32)
    y_want, acc_want = orc.bmm_w8a8(xq, wq, act, ws, True, False, out_bf16=(out == "bf16"))
    y, acc = _run(sq, xq, wq, act, ws, True, False, out)
    assert acc[0, 0, 0] == K * 16384 and acc[1, 0, 5] == -K * 16256
    assert_bits_equal(acc, acc_want, "acc")
    assert_bits_equal(y, y_want, "y")


def test_bmm_attention_sizes_match_per_batch_gemm(sq):
    """OPT-6.7B-shaped attention (32 heads, 2048 tokens, head dimension 128):
    one batched launch equals 32 separate GEMM calls, bit for bit, for the
    scores and for P V."""
    H, T, D = 32, 2048, 128
    g = torch.Generator(device="cuda").manual_seed(5)
    for (M, N, K) in [(T, T, D), (T, D, T)]:
        xq = torch.randint(-127, 128, (H, M, K), dtype=torch.int8, device="cuda", generator=g)
        wq = torch.randint(-127, 128, (H, N, K), dtype=torch.int8, device="cuda", generator=g)
        act = torch.rand(H * M, device="cuda", generator=g) * 0.01 + 1e-4
        ws = torch.rand(H, device="cuda", generator=g) * 0.01 + 1e-4
        y = torch.empty((H, M, N), dtype=torch.bfloat16, device="cuda")
        sq.sq_bmm_w8a8(xq, wq, act, ws, y, per_token=True, w_per_channel=False)
        ref = torch.empty_like(y)
        ws_h = ws.repeat_interleave(N)
        for h in range(H):
            sq.sq_gemm_w8a8(xq[h], wq[h], act[h * M:(h + 1) * M], ws_h[h * N:(h + 1) * N], ref[h],
                            workspace=sq.Workspace())
        sq.sq_sync_status()
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
