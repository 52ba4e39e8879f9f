"""GPU parity of the tcgen05 INT8 GEMM + dequantizing epilogue against the
oracle: INT32 accumulators and outputs (fp32 and bf16) bit for bit, on tiny
ragged shapes, multi-tile shapes with ragged tails, and the int8 extremes."""
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


def _operands(M, N, K, seed):
    r = np.random.default_rng(seed)
    xq = r.integers(-127, 128, (M, K)).astype(np.int8)
    wq = r.integers(-127, 128, (N, K)).astype(np.int8)
    act = r.uniform(1e-3, 0.1, M).astype(np.float32)
    ws = r.uniform(1e-4, 1e-2, N).astype(np.float32)
    return xq, wq, act, ws


def _run(sq, xq, wq, act, ws, per_token, out, acc=True, workspace=None):
    M, N = xq.shape[0], wq.shape[0]
    y = torch.empty((M, N), dtype=torch.bfloat16 if out == "bf16" else torch.float32,
                    device="cuda")
    a = torch.empty((M, N), dtype=torch.int32, device="cuda") if acc else None
    act_d = dev(act if per_token else act[:1])
    sq.sq_gemm_w8a8(dev(xq), dev(wq), act_d, dev(ws), y, per_token=per_token, acc_out=a,
                    workspace=workspace)
    sq.sq_sync_status()
    return host(y), (host(a) if acc else None)


SHAPES = [(1, 1, 16), (3, 17, 48), (17, 255, 1040), (128, 256, 128), (129, 257, 144),
          (255, 300, 4096), (1, 4096, 4096), (8, 1000, 2064), (200, 512, 272),
          (384, 768, 256)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_gemm_small_shapes(sq, orc, M, N, K, out):
    xq, wq, act, ws = _operands(M, N, K, M * 131 + N * 7 + K)
    y_want, acc_want = orc.gemm_w8a8(xq, wq, act, ws, per_token=True, out_bf16=(out == "bf16"))
    y, acc = _run(sq, xq, wq, act, ws, True, out, workspace=sq.Workspace())
    assert_bits_equal(acc, acc_want, "acc")
    assert_bits_equal(y, y_want, "y")


@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_gemm_per_tensor_scale(sq, orc, out):
    M, N, K = 70, 130, 512
    xq, wq, act, ws = _operands(M, N, K, 99)
    y_want, acc_want = orc.gemm_w8a8(xq, wq, act[:1], ws, per_token=False,
                                     out_bf16=(out == "bf16"))
    y, acc = _run(sq, xq, wq, act, ws, False, out, workspace=sq.Workspace())
    assert_bits_equal(acc, acc_want, "acc")
    assert_bits_equal(y, y_want, "y")


def test_gemm_extremes(sq, orc):
    """+-127 everywhere at the largest K of the workloads (20480): the INT32
    accumulators reach +-330,321,920 exactly."""
    M, N, K = 130, 260, 20480
    xq = np.full((M, K), 127, np.int8)
    wq = np.full((N, K), 127, np.int8)
    wq[1::2] = -127
    xq[5, ::2] = -127
    act = np.full(M, 0.01, np.float32)
    ws = np.full(N, 0.001, np.float32)
    y_want, acc_want = orc.gemm_w8a8(xq, wq, act, ws)
    y, acc = _run(sq, xq, wq, act, ws, True, "f32", workspace=sq.Workspace())
    assert acc[0, 0] == 330321920 and acc[0, 1] == -330321920
    assert_bits_equal(acc, acc_want, "acc")
    assert_bits_equal(y, y_want, "y")


@pytest.mark.parametrize("M,N,K", [(200, 264, 240), (200, 264, 256), (200, 264, 272),
                                   (200, 264, 512), (200, 264, 528), (2048, 2048, 128)])
def test_gemm_short_k_epilogue(sq, orc, M, N, K):
    """Short K (at most four 128-byte k-blocks) runs the epilogue on three
    warps per accumulator quarter, each taking every third 32-column chunk;
    K = 528 is the first width back on one warp per quarter.  The largest
    accumulators the codes allow (-128 x -128 x K) sit beside random rows:
    2^22 at K = 256, past the 2^22 bound of fp32 integer tricks at K = 272
    (the conversion must stay exact there too).  2048 x 2048 picks the 256-column tile, the others the 192-column one."""
    r = np.random.default_rng(K + N)
    xq = r.integers(-128, 128, (M, K)).astype(np.int8)
    wq = r.integers(-128, 128, (N, K)).astype(np.int8)
    xq[:3] = -128
    wq[:2] = -128
    wq[2] = 127
    act = r.uniform(1e-3, 0.1, M).astype(np.float32)
    ws = r.uniform(1e-4, 1e-2, N).astype(np.float32)
    y_want, acc_want = orc.gemm_w8a8(xq, wq, act, ws, out_bf16=True)
    y, acc = _run(sq, xq, wq, act, ws, True, "bf16", workspace=sq.Workspace())
    assert acc[0, 0] == K * 16384 and acc[0, 2] == -K * 16256
    assert_bits_equal(acc, acc_want, "acc")
    assert_bits_equal(y, y_want, "y")


# Shapes on the CTA-pair kernel (more than 128 tokens, more than four
# k-blocks): 256-row tiles shared by two CTAs, each CTA holding 128 rows of A
# and half the tile's rows of B.  Tokens within one pair tile (the odd CTA's
# rows partly or wholly past M), ragged rows and columns, odd N (direct
# stores), both tile widths (192 when every tile fits in one wave, 256 for
# 2048 x 4096), and more tiles than pairs (the persistent loop wraps).
PAIR_SHAPES = [(129, 257, 1040), (200, 300, 640), (256, 256, 1024), (257, 200, 2048),
               (1000, 777, 640), (2048, 4096, 1024), (4100, 1000, 640)]


@pytest.mark.parametrize("M,N,K", PAIR_SHAPES)
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_gemm_cta_pair_shapes(sq, orc, M, N, K, out):
    xq, wq, act, ws = _operands(M, N, K, M * 13 + N * 5 + K)
    rows = None
    if M * N * K > 1 << 31:  # sampled rows (every column) for the large ones
        r = np.random.default_rng(M + K)
        rows = np.unique(np.concatenate([
            [0, 1, 127, 128, 255, 256, M // 2, M - 2, M - 1],
            r.integers(0, M, 24)]).clip(0, M - 1)).astype(np.int64)
    y_want, acc_want = orc.gemm_w8a8(xq, wq, act, ws, per_token=True, rows=rows,
                                     out_bf16=(out == "bf16"))
    y, acc = _run(sq, xq, wq, act, ws, True, out, workspace=sq.Workspace())
    if rows is not None:
        y, acc = y[rows], acc[rows]
    assert_bits_equal(acc, acc_want, "acc")
    assert_bits_equal(y, y_want, "y")


def test_gemm_without_acc_dump(sq, orc):
    M, N, K = 300, 520, 1024
    xq, wq, act, ws = _operands(M, N, K, 5)
    y_want, _ = orc.gemm_w8a8(xq, wq, act, ws, out_bf16=True)
    y, _ = _run(sq, xq, wq, act, ws, True, "bf16", acc=False, workspace=sq.Workspace())
    assert_bits_equal(y, y_want, "y")


def test_gemm_is_deterministic(sq):
    M, N, K = 515, 1030, 2048
    xq, wq, act, ws = _operands(M, N, K, 6)
    ws_buf = sq.Workspace()
    y1, a1 = _run(sq, xq, wq, act, ws, True, "bf16", workspace=ws_buf)
    y2, a2 = _run(sq, xq, wq, act, ws, True, "bf16", workspace=ws_buf)
    assert_bits_equal(a1, a2, "acc rerun")
    assert_bits_equal(y1, y2, "y rerun")


# ---------------------------------------------------------------- small M
# Up to 8 tokens, and up to 128 on outputs too narrow for the large-M tiles
# to fill the SMs, take the stream-K weight-streaming kernel: tokens padded to
# 8/16/32/64/128 as the MMA N dimension, (tile, k-block) units split evenly
# over the SMs, partial tiles summed exactly by the last CTA to arrive.  The
# wide outputs below (49152 and 57344 columns at 9 to 128 tokens) run the
# large-M kernel with a single, mostly padded, 128-row block.
SMALL_SHAPES = [
    (1, 130, 16), (2, 1000, 12288), (8, 4096, 2064), (9, 300, 4096), (16, 2048, 1040),
    (17, 777, 8192), (32, 1024, 6144), (33, 260, 144), (64, 3000, 2048), (100, 1536, 4096),
    (128, 512, 12288), (128, 49152, 256), (5, 128, 20480), (16, 49152, 512),
    (12, 57344, 384), (8, 49152, 384),
]


@pytest.mark.parametrize("M,N,K", SMALL_SHAPES)
def test_gemm_small_m_stream_k(sq, orc, M, N, K):
    xq, wq, act, ws = _operands(M, N, K, M * 7 + N * 3 + K)
    for out in ("bf16", "f32"):
        y_want, acc_want = orc.gemm_w8a8(xq, wq, act, ws, per_token=True,
                                         out_bf16=(out == "bf16"))
        y, acc = _run(sq, xq, wq, act, ws, True, out, workspace=sq.Workspace())
        assert_bits_equal(acc, acc_want, f"acc {out}")
        assert_bits_equal(y, y_want, f"y {out}")


def test_gemm_small_m_workspace_reuse(sq, orc):
    """One workspace buffer reused across shapes, holding garbage from the
    previous call: the kernel needs no particular initial contents."""
    wsbuf = torch.full((64 << 20,), 0x5A, dtype=torch.uint8, device="cuda")
    for (M, N, K) in [(128, 2000, 4096), (3, 50000, 1024), (64, 7000, 2048), (1, 1000, 12288)]:
        need = sq.sq_gemm_workspace_bytes(M, N, K)
        assert 0 < need <= wsbuf.numel()
        xq, wq, act, ws = _operands(M, N, K, M + N + K)
        y_want, acc_want = orc.gemm_w8a8(xq, wq, act, ws, out_bf16=True)
        y, acc = _run(sq, xq, wq, act, ws, True, "bf16", workspace=wsbuf)
        assert_bits_equal(acc, acc_want, "acc reuse")
        assert_bits_equal(y, y_want, "y reuse")


def test_gemm_decode_path_choice(sq):
    """Which decode shapes need the stream-K scratch: up to 8 tokens always;
    9 to 128 tokens only while the large-M tiles across N would not give
    every SM one; more than 128 never."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert sq.sq_gemm_workspace_bytes(8, 49152, 12288) > 0
    assert sq.sq_gemm_workspace_bytes(16, 49152, 12288) == 0  # 256 tiles of 192
    assert sq.sq_gemm_workspace_bytes(128, 49152, 12288) == 0
    assert sq.sq_gemm_workspace_bytes(128, 12288, 12288) > 0  # 64 tiles
    assert sq.sq_gemm_workspace_bytes(16, 192 * (sms - 1), 4096) > 0
    assert sq.sq_gemm_workspace_bytes(129, 512, 4096) == 0


def test_gemm_small_m_rejects_short_workspace(sq):
    M, N, K = 8, 1024, 1024
    xq, wq, act, ws = _operands(M, N, K, 1)
    need = sq.sq_gemm_workspace_bytes(M, N, K)
    short = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sq.SQError) as ei:
        sq.sq_gemm_w8a8(dev(xq), dev(wq), dev(act), dev(ws), y, workspace=short)
    assert ei.value.status == 8  # SQ_ERR_WORKSPACE


# Shapes for the bias epilogue: large-M tiles with the TMA-store epilogue
# (N a multiple of 8), with direct stores (N % 8 != 0), fp32 and bf16 out,
# and the stream-K weight-streaming path (few tokens on narrow outputs).
BIAS_SHAPES = [(300, 512, 1040), (257, 300, 272), (1024, 2048, 512), (1, 4096, 4096),
               (33, 1000, 2064), (128, 520, 1024)]


@pytest.mark.parametrize("M,N,K", BIAS_SHAPES)
@pytest.mark.parametrize("out", ["f32", "bf16"])
@pytest.mark.parametrize("per_token", [True, False])
def test_gemm_bias(sq, orc, M, N, K, out, per_token):
    """y = dequantized accumulator + bias[n], bit for bit against the oracle
    (sampled rows for the larger shapes, every column)."""
    xq, wq, act, ws = _operands(M, N, K, M * 17 + N * 3 + K)
    bias = np.random.default_rng(M + N).normal(0, 0.5, N).astype(np.float32)
    act_used = act if per_token else act[:1]
    rows = np.unique(np.array([0, 1, 127, 128, M // 2, M - 1]).clip(0, M - 1)).astype(np.int64)
    y_want, acc_want = orc.gemm_w8a8(xq, wq, act_used, ws, per_token=per_token, rows=rows,
                                     out_bf16=(out == "bf16"), bias=bias)
    y = torch.empty((M, N), dtype=torch.bfloat16 if out == "bf16" else torch.float32,
                    device="cuda")
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    sq.sq_gemm_w8a8(dev(xq), dev(wq), dev(act_used), dev(ws), y, per_token=per_token,
                    acc_out=acc, workspace=sq.Workspace(), bias=dev(bias))
    sq.sq_sync_status()
    r = torch.from_numpy(rows).cuda()
    assert_bits_equal(host(acc[r]), acc_want, "acc")
    assert_bits_equal(host(y[r]), y_want, "y")


def test_gemm_zero_bias_is_no_bias(sq):
    """A zero bias leaves every output bit unchanged (both paths)."""
    for M, N, K in [(300, 512, 1040), (8, 1000, 2064)]:
        xq, wq, act, ws = [dev(v) for v in _operands(M, N, K, 99)]
        y0 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        y1 = torch.empty_like(y0)
        sq.sq_gemm_w8a8(xq, wq, act, ws, y0, workspace=sq.Workspace())
        sq.sq_gemm_w8a8(xq, wq, act, ws, y1, workspace=sq.Workspace(),
                        bias=torch.zeros(N, dtype=torch.float32, device="cuda"))
        sq.sq_sync_status()
        assert torch.equal(y0.view(torch.int16), y1.view(torch.int16))
