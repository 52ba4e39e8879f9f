"""Shared test helpers: moving the seeded numpy inputs onto the GPU and
comparing results.  No arithmetic of the method lives here."""
from __future__ import annotations

import numpy as np
import torch


def dev(a: np.ndarray | None, dtype: str = "f32"):
    """numpy (fp32, or bf16 bit patterns in uint16, or int8) -> CUDA tensor."""
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    """CUDA tensor -> numpy (bf16 as uint16 bit patterns)."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def assert_bits_equal(got: np.ndarray, want: np.ndarray, what: str):
    got = np.ascontiguousarray(got)
    want = np.ascontiguousarray(want)
    assert got.shape == want.shape, f"{what}: shape {got.shape} != {want.shape}"
    if got.dtype.kind == "f":
        g = got.view(np.uint32 if got.itemsize == 4 else np.uint64)
        w = want.view(np.uint32 if want.itemsize == 4 else np.uint64)
    else:
        g, w = got, want
    bad = np.flatnonzero(g.reshape(-1) != w.reshape(-1))
    if bad.size:
        i = bad[0]
        raise AssertionError(
            f"{what}: {bad.size} of {g.size} elements differ; first at flat index {i}: "
            f"got {got.reshape(-1)[i]!r} want {want.reshape(-1)[i]!r}")


def ulp_diff_f32(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """|a - b| in units of fp32 ulps (both finite, same sign expected)."""
    ai = np.ascontiguousarray(a, np.float32).view(np.int32).astype(np.int64)
    bi = np.ascontiguousarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(ai - bi)
