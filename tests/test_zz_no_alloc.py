"""sq_gemm_w8a8_noalloc: the INT8 GEMM for callers that cannot allocate
device memory (an engine or framework that owns every allocation and forbids
new ones while it runs, or a plugin hook that only receives its inputs and
outputs).  Its scratch is a fixed 8 MiB device array inside the library, so
the caller passes no workspace.

Each case calls the entry point twice in a row through the C ABI and checks
both results bit for bit against sq_gemm_w8a8 (with a caller workspace) on
the same inputs -- the tolerance every other GEMM test uses.  The file sorts
last so that a run stopping at its first failure has run every other test
before it; it also passes when run on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

STATIC_SCRATCH_BYTES = 8 << 20


@pytest.fixture(scope="module")
def sq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import w8a8_int8_gemm_calib_b200 as m

    return m


def _inputs(M, N, K, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    xq = torch.randint(-127, 128, (M, K), dtype=torch.int8, device="cuda", generator=g)
    wq = torch.randint(-127, 128, (N, K), dtype=torch.int8, device="cuda", generator=g)
    act = torch.rand(M, device="cuda", generator=g) * 0.1 + 1e-3
    ws = torch.rand(N, device="cuda", generator=g) * 0.01 + 1e-4
    return xq, wq, act, ws


def _noalloc(sq, xq, wq, act, ws, y, acc, per_token=True):
    M, K = xq.shape
    N = wq.shape[0]
    st = torch.cuda.current_stream().cuda_stream
    dt = sq.SQ_BF16 if y.dtype == torch.bfloat16 else sq.SQ_F32
    return sq.lib.sq_gemm_w8a8_noalloc(
        xq.data_ptr(), wq.data_ptr(), M, N, K, act.data_ptr(), int(per_token), ws.data_ptr(),
        y.data_ptr(), dt, acc.data_ptr() if acc is not None else None, ctypes.c_void_p(st))


@pytest.mark.parametrize("M,N,K,out", [
    (1, 49152, 12288, torch.bfloat16),   # decode shape: weight-streaming path
    (8, 4096, 4096, torch.float32),
    (33, 1000, 2064, torch.bfloat16),    # stream-K splits tiles across SMs
    (300, 520, 1024, torch.bfloat16),    # M > 128: needs no scratch at all
])
def test_noalloc_matches_workspace_entry_point(sq, M, N, K, out):
    assert sq.sq_gemm_workspace_bytes(M, N, K) <= STATIC_SCRATCH_BYTES
    xq, wq, act, ws = _inputs(M, N, K, M + N + K)
    y_ref = torch.empty((M, N), dtype=out, device="cuda")
    a_ref = torch.empty((M, N), dtype=torch.int32, device="cuda")
    sq.sq_gemm_w8a8(xq, wq, act, ws, y_ref, acc_out=a_ref, workspace=sq.Workspace())
    sq.sq_sync_status()
    for _ in range(2):  # two calls in a row share the static scratch
        y = torch.full((M, N), float("nan"), dtype=out, device="cuda")
        acc = torch.zeros((M, N), dtype=torch.int32, device="cuda")
        assert _noalloc(sq, xq, wq, act, ws, y, acc) == 0, sq._lib.last_error()
        sq.sq_sync_status()
        assert torch.equal(acc, a_ref)
        assert torch.equal(y.view(torch.int16 if out == torch.bfloat16 else torch.int32),
                           y_ref.view(torch.int16 if out == torch.bfloat16 else torch.int32))


def test_noalloc_refuses_shapes_beyond_its_scratch(sq):
    """A shape whose scratch exceeds the 8 MiB array is refused before any
    launch, with a message that names the sizes (128 tokens on a 12288-wide
    output: 64 large-M tiles would not fill the SMs, so it stays on the
    stream-K path and its scratch)."""
    M, N, K = 128, 12288, 12288
    assert sq.sq_gemm_workspace_bytes(M, N, K) > STATIC_SCRATCH_BYTES
    xq, wq, act, ws = _inputs(M, N, 256, 7)[0], None, None, None
    xq = torch.zeros((M, K), dtype=torch.int8, device="cuda")
    wq = torch.zeros((N, K), dtype=torch.int8, device="cuda")
    act = torch.ones(M, device="cuda")
    ws = torch.ones(N, device="cuda")
    y = torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda")
    st = _noalloc(sq, xq, wq, act, ws, y, None)
    assert st == 8  # SQ_ERR_WORKSPACE
    assert "static scratch" in sq._lib.last_error()
    sq.sq_sync_status()
    assert bool((y == 3.0).all())  # nothing was launched


def test_noalloc_boundary_on_the_stream_k_path(sq):
    """At the edge of the 8 MiB array: on a stream-K shape whose units cover
    every SM (1000 output channels, K = 12288), the largest token count whose
    scratch fits (55 at 148 SMs: 256 + 148 * 2 * 55 * 128 * 4 bytes) is
    served -- twice, bit-exact against the workspace entry point -- and one
    token more is refused before any launch."""
    N, K = 1000, 12288
    fits = [m for m in range(9, 129)
            if 0 < sq.sq_gemm_workspace_bytes(m, N, K) <= STATIC_SCRATCH_BYTES]
    M = max(fits)
    assert sq.sq_gemm_workspace_bytes(M + 1, N, K) > STATIC_SCRATCH_BYTES
    xq, wq, act, ws = _inputs(M + 1, N, K, 11)
    y_ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    a_ref = torch.empty((M, N), dtype=torch.int32, device="cuda")
    sq.sq_gemm_w8a8(xq[:M], wq, act[:M], ws, y_ref, acc_out=a_ref, workspace=sq.Workspace())
    sq.sq_sync_status()
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        acc = torch.zeros((M, N), dtype=torch.int32, device="cuda")
        assert _noalloc(sq, xq[:M], wq, act[:M], ws, y, acc) == 0, sq._lib.last_error()
        sq.sq_sync_status()
        assert torch.equal(acc, a_ref)
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    y = torch.full((M + 1, N), 3.0, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(sq, xq, wq, act, ws, y, None) == 8  # SQ_ERR_WORKSPACE
    sq.sq_sync_status()
    assert bool((y == 3.0).all())
