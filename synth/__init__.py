"""Seeded synthetic inputs for the smoothed W8A8 linear layer.

This module only draws random numbers and casts them to the storage dtype;
it holds none of the method's arithmetic.  Both the CUDA path (through
``bench.py`` and the GPU tests) and the CPU oracle consume the same arrays.

Value recipe (the activation-outlier structure described in
"嵌入式 SLM 动态权重量化：SmoothQuant 激活异常值迁移与 INT8 部署实战" §一.1 and
"SmoothQuant：大型语言模型的精准高效训练后量化 — 深度技术评审" §4, observation 3):

* ordinary activation entries ~ N(0, 1);
* a fixed set of outlier channels -- ``round(p * K)`` of them, picked by a
  seeded permutation -- whose entries are multiplied by a per-channel factor
  ``c_j ~ U(50, 120)``; the channels and factors are the same for the
  calibration tokens and the runtime tokens (outliers persist per channel);
* weights ~ N(0, sigma) with sigma the standard deviation the workload names;
* LayerNorm gamma ~ 1 + N(0, 0.1), beta ~ N(0, 0.02);
* bf16 tensors are drawn in fp32 and rounded to nearest even.

Every tensor has its own PCG64 sub-stream keyed by (seed, tensor name).
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import zlib
from dataclasses import dataclass, field

import numpy as np

ROWS_PER_BLOCK = 256  # rows drawn per sub-stream (independent of thread count)


def rng_for(seed: int, name: str, block: int = 0) -> np.random.Generator:
    """Independent PCG64 stream for one named tensor (and row block) of one
    workload."""
    return np.random.Generator(np.random.PCG64([seed, zlib.crc32(name.encode()), block]))


def _normal_rows(seed: int, name: str, T: int, K: int) -> np.ndarray:
    """[T, K] fp32 N(0,1), drawn in blocks of ROWS_PER_BLOCK rows, each from
    its own sub-stream, on a thread pool (numpy releases the GIL)."""
    x = np.empty((T, K), dtype=np.float32)
    nb = (T + ROWS_PER_BLOCK - 1) // ROWS_PER_BLOCK

    def fill(b):
        r0 = b * ROWS_PER_BLOCK
        r1 = min(T, r0 + ROWS_PER_BLOCK)
        rng_for(seed, name, b).standard_normal((r1 - r0, K), dtype=np.float32, out=x[r0:r1])

    with cf.ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
        list(ex.map(fill, range(nb)))
    return x


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest even) and return the raw uint16 patterns.
    (Inputs are finite: the generators draw no NaN.)"""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    out = np.empty(u.shape, dtype=np.uint16)
    flat_u, flat_o = u.reshape(-1), out.reshape(-1)
    step = 1 << 24

    def conv(i):
        v = flat_u[i:i + step]
        flat_o[i:i + step] = ((v + (np.uint32(0x7FFF) + ((v >> 16) & 1))) >> 16).astype(np.uint16)

    with cf.ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
        list(ex.map(conv, range(0, flat_u.size, step)))
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (exact)."""
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class Outliers:
    channels: np.ndarray  # int64 channel indices
    factors: np.ndarray   # float32 multipliers, one per channel


def outlier_pattern(seed: int, K: int, frac: float = 0.0, count: int | None = None,
                    tag: str = "x") -> Outliers:
    n = int(round(frac * K)) if count is None else int(count)
    r = rng_for(seed, f"outliers/{tag}")
    ch = np.sort(r.permutation(K)[:n]).astype(np.int64)
    fac = r.uniform(50.0, 120.0, size=n).astype(np.float32)
    return Outliers(ch, fac)


def activations(seed: int, name: str, T: int, K: int, out: Outliers,
                relu: bool = False) -> np.ndarray:
    """[T, K] fp32 activations with persistent outlier channels."""
    x = _normal_rows(seed, name, T, K)
    if out.channels.size:
        x[:, out.channels] *= out.factors[None, :]
    if relu:
        np.maximum(x, 0.0, out=x)
    return x


def weights(seed: int, name: str, N: int, K: int, sigma: float) -> np.ndarray:
    w = _normal_rows(seed, name, N, K)
    w *= np.float32(sigma)
    return w


def ln_params(seed: int, name: str, K: int):
    r = rng_for(seed, name)
    gamma = (1.0 + 0.1 * r.standard_normal(K)).astype(np.float32)
    beta = (0.02 * r.standard_normal(K)).astype(np.float32)
    return gamma, beta


# ----------------------------------------------------------------- workloads

@dataclass
class Linear:
    """One smoothed linear: X[T,K] -> Y[T,N] with its calibration set."""
    name: str
    K: int
    N: int
    T: int             # runtime tokens
    T_cal: int         # calibration tokens
    ln: bool           # a LayerNorm precedes the linear
    alpha: float
    per_token: bool    # dynamic per-token (True) or static per-tensor (False)
    dtype: str         # "f32" or "bf16" for X, W and Y
    w_sigma: float
    outlier_frac: float = 0.0
    outlier_count: int | None = None
    relu_input: bool = False
    seed: int = 1000
    shared: str | None = None  # linears with the same key share W, LN and calibration data


@dataclass
class Workload:
    name: str
    description: str
    linears: list = field(default_factory=list)


def workloads() -> dict:
    """The five workloads, named by what they are with their sizes."""
    w = {}
    w["tiny_k1024"] = Workload(
        "tiny_k1024",
        "single smoothed linear, fp32, K=N=1024, 512 calibration + 128 runtime "
        "tokens, 4 outlier channels, LayerNorm, alpha 0.5, static per-tensor",
        [Linear("linear", 1024, 1024, 128, 512, True, 0.5, False, "f32", 0.02,
                outlier_count=4, seed=1000)])
    w["opt6.7b_qkv_t2048"] = Workload(
        "opt6.7b_qkv_t2048",
        "OPT-6.7B-shaped fused QKV: LayerNorm then 4096->12288 over 2048 tokens, "
        "bf16, 12 outlier channels, 4096 calibration tokens, alpha 0.5, per-token",
        [Linear("qkv", 4096, 12288, 2048, 4096, True, 0.5, True, "bf16", 0.02,
                outlier_count=12, seed=1001)])
    lin13 = []
    for alpha in (0.5, 0.8):
        a = f"a{alpha}"
        lin13 += [
            Linear(f"qkv_{a}", 5120, 15360, 4096, 4096, True, alpha, True, "bf16", 0.02,
                   outlier_frac=0.003, seed=1002),
            Linear(f"out_{a}", 5120, 5120, 4096, 4096, False, alpha, True, "bf16", 0.02,
                   outlier_frac=0.003, seed=1002),
            Linear(f"fc1_{a}", 5120, 20480, 4096, 4096, True, alpha, True, "bf16", 0.02,
                   outlier_frac=0.003, seed=1002),
            Linear(f"fc2_{a}", 20480, 5120, 4096, 4096, False, alpha, True, "bf16", 0.02,
                   outlier_frac=0.003, relu_input=True, seed=1002),
        ]
    w["13b_layer_t4096"] = Workload(
        "13b_layer_t4096",
        "13B-shaped decoder-layer linears, hidden 5120, 4096 tokens, bf16: QKV, "
        "out-proj, fc1, fc2 (ReLU input), alpha 0.5 and 0.8, per-token", lin13)
    w["175b_fc1_decode"] = Workload(
        "175b_fc1_decode",
        "175B-shaped decode fc1 12288->49152, M in {1,8,32,128}, bf16, 0.3% "
        "outlier channels, INT8 weights streamed from HBM, per-token",
        [Linear(f"fc1_m{m}", 12288, 49152, m, 4096, False, 0.5, True, "bf16", 0.02,
                outlier_frac=0.003, seed=1003, shared="fc1") for m in (1, 8, 32, 128)])
    w["large_prefill_k8192"] = Workload(
        "large_prefill_k8192",
        "large prefill: absmax over 65536x8192 bf16 calibration tokens, then "
        "8192->28672 at 16384 tokens, 0.5% outliers, W N(0,0.015), alpha 0.5, "
        "static per-tensor, bf16 out",
        [Linear("mlp", 8192, 28672, 16384, 65536, False, 0.5, False, "bf16", 0.015,
                outlier_frac=0.005, seed=1004)])
    return w


WORKLOAD_ORDER = ["tiny_k1024", "opt6.7b_qkv_t2048", "13b_layer_t4096",
                  "175b_fc1_decode", "large_prefill_k8192"]


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    return x if dtype == "f32" else bf16_bits(x)


def make_linear_inputs(lin: Linear, T: int | None = None, T_cal: int | None = None,
                       N: int | None = None) -> dict:
    """Draw one linear's tensors.  Optional T/T_cal/N shrink the draw (rows of
    the same streams are not preserved across sizes; every size is its own
    seeded draw).  Returns numpy arrays: fp32, or bf16 bit patterns (uint16)."""
    T = lin.T if T is None else T
    T_cal = lin.T_cal if T_cal is None else T_cal
    N = lin.N if N is None else N
    # one outlier pattern per (seed, K): the linears of a layer that share an
    # input width share the channels, as a model's hidden state would
    out = outlier_pattern(lin.seed, lin.K, lin.outlier_frac, lin.outlier_count,
                          tag=f"k{lin.K}")
    d = {"outliers": out}
    key = lin.shared or lin.name
    d["x_cal"] = _store(activations(lin.seed, f"{key}/x_cal", T_cal, lin.K, out,
                                    relu=lin.relu_input), lin.dtype)
    d["x"] = _store(activations(lin.seed, f"{lin.name}/x", T, lin.K, out,
                                relu=lin.relu_input), lin.dtype)
    d["w"] = _store(weights(lin.seed, f"{key}/w", N, lin.K, lin.w_sigma), lin.dtype)
    if lin.ln:
        d["gamma"], d["beta"] = ln_params(lin.seed, f"{key}/ln", lin.K)
    else:
        d["gamma"] = d["beta"] = None
    return d
