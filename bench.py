#!/usr/bin/env python
"""Benchmark of the smoothed W8A8 linear layer (SmoothQuant hot path) on B200.

One step = one pass of the whole path over one batch of synthetic input:
calibration absmax (LayerNorm-fused when a LayerNorm precedes), smoothing
factors (eq. (4)), weight + LayerNorm fold with per-output-channel INT8,
the fused LayerNorm + smoothing + INT8 activation quantizer, and the INT8
tcgen05 GEMM with the dequantizing epilogue.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl reference]

`value` is whole-job throughput in TOPS = 2*M*N*K per step (all ranks) over
the device time of the timed steps, max over ranks.  Each step is one replay
of a CUDA graph of the five calls, timed on the device by event nodes at the
graph's two ends.  The per-call breakdown, taken after the timed steps,
times graphs of the first 1..4 calls the same way: a call's time is what it
adds to the step.  Before every timed replay L2 is flushed outside the timed
events: a 256 MiB buffer is written, then another 256 MiB buffer is read, so
that the timed work finds neither its data nor the flush's dirty lines in
L2.  Inputs are resident in HBM.
`e2e` is the same metric through the public Python API with pinned host
buffers: every step copies its inputs host->device and its output back.
`--impl reference` times the CPU oracle (tests-only code) on bounded samples
of the same workload, each step extrapolated linearly to the full workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "W8A8 smoothed-linear TOPS & % INT8 peak; small-M HBM GB/s (1×B200)"
DEFAULT_WORKLOAD = "opt6.7b_qkv_t2048"
FLUSH_BYTES = 256 << 20
# INT8 dense peak = measured bf16 dense peak x the nominal int8:bf16 ratio
# (4.5 POPS : 2.25 PFLOP/s = 2).
INT8_PER_BF16 = 2.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# DRAM bytes (read + write) of one launch of the dominant kernel, from the ncu
# capture summarised in profiles/ (null when the kernel has changed since)
GEMM_DRAM_TRAFFIC = {
    # the kernel was rebuilt after this capture (template parameters for the
    # short-K and error-mode epilogues; its 4-warp path's loads and stores are
    # the same), so the counters are given as context, not claimed for it
    "opt6.7b_qkv_t2048": (None, "not re-captured for this build; last capture "
                          "(profiles/gemm_w8a8_tc_opt6.7b_qkv_t2048.md, earlier build of the "
                          "same main loop): dram__bytes_read.sum 58.82 MB + dram__bytes_write.sum "
                          "16.51 MB = 75.33 MB per launch"),
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--linear", default=None, help="linear of the workload (default: first)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-small-m", action="store_true",
                    help="skip the decode-shaped (small-M) GEMM measurement")
    return ap.parse_args()


def pick_linear(args):
    wl = synth.workloads()[args.workload]
    lin = wl.linears[0]
    if args.linear:
        lin = next(l for l in wl.linears if l.name == args.linear)
    return wl, lin


def config_of(wl, lin, world):
    return {
        "workload": wl.name,
        "linear": lin.name,
        "M": lin.T, "N": lin.N, "K": lin.K, "T_cal": lin.T_cal,
        "layernorm": lin.ln, "alpha": lin.alpha,
        "act_quant": "per-token dynamic" if lin.per_token else "per-tensor static",
        "io_dtype": lin.dtype,
        "l2": "flushed before every timed step, outside the timed events (256 MiB written, then another 256 MiB read)",
        "timing": "CUDA graph per step, device events at its two ends; per-call times as differences of graphs of the step's first 1..5 calls",
        "parallelism": f"replicas x{world}",
    }


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while the timed region runs."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self._ok = False

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.02)

    def __enter__(self):
        if self._ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self._ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- our arm
class Layer:
    """Device buffers of one smoothed linear and the five calls of one step."""

    def __init__(self, sq, torch, lin, d, dev):
        self.sq, self.torch, self.lin = sq, torch, lin
        f32, bf16 = torch.float32, torch.bfloat16
        io = bf16 if lin.dtype == "bf16" else f32
        K, N, M, Tc = lin.K, lin.N, lin.T, lin.T_cal
        self.io = io

        def t(a):
            if a is None:
                return None
            if a.dtype == np.uint16:
                return torch.from_numpy(a.view(np.int16)).view(bf16).to(dev)
            return torch.from_numpy(a).to(dev)

        self.x_cal, self.x, self.w = t(d["x_cal"]), t(d["x"]), t(d["w"])
        self.gamma, self.beta = t(d["gamma"]), t(d["beta"])
        self.amax = torch.empty(K, dtype=f32, device=dev)
        self.s = torch.empty(K, dtype=f32, device=dev)
        self.inv_s = torch.empty(K, dtype=f32, device=dev)
        self.dA = torch.empty(1, dtype=f32, device=dev)
        self.wq = torch.empty((N, K), dtype=torch.int8, device=dev)
        self.ws = torch.empty(N, dtype=f32, device=dev)
        self.g2 = torch.empty(K, dtype=f32, device=dev) if lin.ln else None
        self.b2 = torch.empty(K, dtype=f32, device=dev) if lin.ln else None
        self.xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        self.act = torch.empty(M if lin.per_token else 1, dtype=f32, device=dev)
        self.y = torch.empty((M, N), dtype=io, device=dev)
        self.workspace = sq.Workspace(dev)
        # this library's kernels per step: calibration peak; column peak +
        # eq. (4) factors; weight fold (which also divides gamma and beta by
        # s); quantizer; GEMM
        self.kernels_per_step = 6

    def step(self, ev=None, upto=5):
        """The first `upto` of the five calls (all five: one step); ev = (start,
        end) events recorded around them, or None.  (Running the weight
        column peaks on a second stream beside the calibration was measured
        no faster: whichever kernel starts first fills the SMs.)"""
        sq, L = self.sq, self.lin
        if ev is not None:
            ev[0].record()
        self.amax.zero_()
        sq.sq_calib_absmax(self.x_cal, self.amax, self.gamma, self.beta, 1e-5)
        if upto >= 2:
            sq.sq_smooth_scales(self.amax, self.w, L.alpha, self.s, self.inv_s,
                                None if L.per_token else self.dA)
        if upto >= 3:
            sq.sq_fuse_weights_q8(self.w, self.s, self.wq, self.ws, self.gamma, self.beta,
                                  self.g2, self.b2)
        act = self.act
        if upto >= 4:
            if not L.per_token:
                act.copy_(self.dA)
            if L.ln:
                sq.sq_ln_smooth_quant_act(self.x, self.xq, act, self.g2, self.b2, 1e-5,
                                          per_token=L.per_token)
            else:
                sq.sq_ln_smooth_quant_act(self.x, self.xq, act, inv_s=self.inv_s,
                                          per_token=L.per_token)
        if upto >= 5:
            sq.sq_gemm_w8a8(self.xq, self.wq, act, self.ws, self.y, per_token=L.per_token,
                            workspace=self.workspace)
        if ev is not None:
            ev[1].record()


class L2Flush:
    """Evicts L2 between timed iterations: writes a buffer twice the L2 size,
    then reads another one, so that L2 holds clean lines of neither inputs
    nor outputs and the timed work pays no write-back of the flush."""

    def __init__(self, torch, dev):
        self.w = torch.empty(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
        self.r = torch.zeros(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    def __call__(self, i):
        self.w.fill_(i)
        self.sink = self.r.max()


def max_over_ranks(value: float, world: int, device) -> float:
    """Largest value over all ranks (every rank gets it).  Used for the timed
    milliseconds: the job is as slow as its slowest rank."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput_tops(ops_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job TOPS: every rank ran `steps` steps of `ops_per_step` ops."""
    return world * ops_per_step * steps / (max_ms * 1e-3) / 1e12


def algorithmic_bytes(lin):
    """Bytes each step reads/writes once (the per-kernel roofline numerators)."""
    b = 2 if lin.dtype == "bf16" else 4
    M, N, K, Tc = lin.T, lin.N, lin.K, lin.T_cal
    return {
        "calib_absmax": Tc * K * b + 4 * K + (8 * K if lin.ln else 0),
        "smooth_scales": N * K * b + 12 * K,
        "fuse_weights_q8": N * K * b + N * K + 4 * N + 4 * K + (16 * K if lin.ln else 0),
        "ln_smooth_quant_act": M * K * b + M * K + 4 * M + (8 * K if lin.ln else 4 * K),
        "gemm_w8a8": M * K + N * K + M * N * b + 4 * N + 4 * M,
    }


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=dev)
    import w8a8_int8_gemm_calib_b200 as sq

    wl, lin = pick_linear(args)
    d = synth.make_linear_inputs(lin)
    layer = Layer(sq, torch, lin, d, dev)
    flush = L2Flush(torch, dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        layer.step()
    sq.sq_sync_status()
    names = ["calib_absmax", "smooth_scales", "fuse_weights_q8", "ln_smooth_quant_act",
             "gemm_w8a8"]

    def capture(upto):
        ev = (torch.cuda.Event(enable_timing=True, external=True),
              torch.cuda.Event(enable_timing=True, external=True))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            layer.step(ev, upto)
        return g, ev

    # the timed graph: one whole step (five calls, six kernels), event
    # nodes only at its two ends
    graph, ev_step = capture(5)
    for _ in range(max(3, args.warmup)):
        graph.replay()
    barrier()

    K = args.steps
    step_ms = []
    clocks = ClockSampler(torch.cuda.current_device())
    with clocks:
        barrier()
        for i in range(K):
            flush(i)  # evicts the previous step's data from L2
            graph.replay()
            torch.cuda.synchronize()
            step_ms.append(ev_step[0].elapsed_time(ev_step[1]))
        barrier()
    sq.sq_sync_status()
    total_ms = max_over_ranks(float(sum(step_ms)), world, dev)
    ops = 2.0 * lin.T * lin.N * lin.K
    value = throughput_tops(ops, K, world, total_ms)

    # per-call breakdown (after the timed region): graphs of the first 1..4
    # calls, timed like the step; a call's time is what it adds to the step
    prefix_ms = {5: statistics.mean(step_ms)}
    for upto in range(1, 5):
        g, ev = capture(upto)
        g.replay()
        t = []
        for i in range(K):
            flush(i)
            g.replay()
            torch.cuda.synchronize()
            t.append(ev[0].elapsed_time(ev[1]))
        prefix_ms[upto] = statistics.mean(t)
        del g
    prefix_ms[0] = 0.0
    per = {n: prefix_ms[j + 1] - prefix_ms[j] for j, n in enumerate(names)}
    sq.sq_sync_status()

    # ---- e2e through the public API with pinned host buffers
    e2e = run_e2e(sq, torch, layer, lin, d, dev, args.e2e_steps, world, barrier)
    small_m = None if args.no_small_m else run_small_m(sq, torch, dev, flush)
    next_rows = {"o2_per_tensor_dynamic_quant": run_o2(sq, torch, layer, lin, flush),
                 "gemm_bias_epilogue": run_gemm_bias(sq, torch, layer, lin, flush),
                 "rmsnorm_quant_per_token": run_rms_quant(sq, torch, layer, lin, flush),
                 "alpha_sweep": run_alpha_sweep(sq, torch, layer, lin, flush),
                 "attention_bmm": run_attention_bmm(sq, torch, layer.x.device, flush)}

    peaks, peak_kind = load_peaks()
    bf16_peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    int8_peak = bf16_peak * INT8_PER_BF16
    gemm_ms = per["gemm_w8a8"]
    gemm_tops = ops / (gemm_ms * 1e-3) / 1e12
    ab = algorithmic_bytes(lin)
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    kernels = {}
    for n in names:
        ms = per[n]
        k = {"ms": round(ms, 5), "gbs": round(ab[n] / (ms * 1e-3) / 1e9, 1),
             "hbm_frac": round(ab[n] / (ms * 1e-3) / 1e9 / hbm, 3)}
        if n == "gemm_w8a8":
            k["tops"] = round(gemm_tops, 1)
            k["int8_frac"] = round(gemm_tops / int8_peak, 3)
        kernels[n] = k
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": K,
        "warmup": max(3, args.warmup),
        "ms_per_step": round(total_ms / K, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8",
        "data": "synthetic (seeded outlier-structured activations, random-init weights)",
        "config": config_of(wl, lin, world),
        "roofline": {
            "bound": "tensor",
            "kernel": "gemm_w8a8 (tcgen05.mma kind::i8)",
            "achieved": round(gemm_tops, 1),
            "peak": round(int8_peak, 1),
            "unit": "TFLOP/s",
            "frac": round(gemm_tops / int8_peak, 4),
            "traffic": GEMM_DRAM_TRAFFIC.get(wl.name, (None, None))[0],
            "traffic_source": GEMM_DRAM_TRAFFIC.get(wl.name, (None, None))[1],
            "peak_note": f"int8 dense = {peak_kind} bf16 burst {bf16_peak} TFLOP/s x 2 "
                         "(nominal int8:bf16 ratio); 'TFLOP/s' here counts int8 ops",
        },
        "kernels": kernels,
        "small_m_decode": small_m,
        "next_rows": next_rows,
        "e2e": e2e,
        "gpu_launches": layer.kernels_per_step * K,
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(lin, d)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_small_m(sq, torch, dev, flush, reps=20):
    """The metric's small-M half: the INT8 GEMM of the 175B-shaped decode fc1
    (K=12288 -> N=49152) at M = 1, 8, 32, 128 tokens, per-token scales, bf16
    out, on seeded random INT8 operands (604 MB of weights streamed from HBM
    each call).  One CUDA-graph replay per call, L2 flushed before each,
    device events around it; GB/s = algorithmic bytes / time."""
    lin = next(l for l in synth.workloads()["175b_fc1_decode"].linears)
    N, K = lin.N, lin.K
    g = torch.Generator(device=dev).manual_seed(1003)
    wq = torch.randint(-127, 128, (N, K), dtype=torch.int8, device=dev, generator=g)
    ws = torch.rand(N, device=dev, generator=g) * 1e-3 + 1e-5
    hbm = load_peaks()[0].get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    out = {"workload": "175b_fc1_decode: fc1 12288->49152, per-token, bf16 out",
           "kernel": "gemm_w8a8 (tcgen05 kind::i8): stream-K weight streaming up to 8 tokens, "
                     "the persistent 128-row-tile kernel beyond (its 256 tiles fill the SMs)",
           "hbm_peak_gbs": hbm}
    for M in (1, 8, 32, 128):
        xq = torch.randint(-127, 128, (M, K), dtype=torch.int8, device=dev, generator=g)
        act = torch.rand(M, device=dev, generator=g) * 1e-2 + 1e-4
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        wsp = sq.Workspace(dev)
        for _ in range(3):
            sq.sq_gemm_w8a8(xq, wq, act, ws, y, workspace=wsp)
        e0 = torch.cuda.Event(enable_timing=True, external=True)
        e1 = torch.cuda.Event(enable_timing=True, external=True)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            e0.record()
            sq.sq_gemm_w8a8(xq, wq, act, ws, y, workspace=wsp)
            e1.record()
        times = []
        for i in range(reps):
            flush(i)
            graph.replay()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        sq.sq_sync_status()
        ms = statistics.mean(times)
        nbytes = M * K + N * K + M * N * 2 + 4 * N + 4 * M
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[f"M{M}"] = {"us": round(ms * 1e3, 2), "gbs": round(gbs, 1),
                        "hbm_frac": round(gbs / hbm, 3), "bytes": int(nbytes),
                        "path": "stream-K" if sq.sq_gemm_workspace_bytes(M, N, K) else "tiles"}
        del graph
    return out


def run_o2(sq, torch, layer, lin, flush, reps=20):
    """Per-tensor dynamic activation quantization (SmoothQuant-O2) on the
    step's activations: one step from the peak of the whole call, two passes
    over x.  One CUDA-graph replay per call, L2 flushed before each, device
    events around it; GB/s over the algorithmic bytes (x read once, codes
    written once), so the second read of x shows as a lower fraction."""
    M, K = lin.T, lin.K
    b = 2 if lin.dtype == "bf16" else 4
    act = torch.empty(1, dtype=torch.float32, device=layer.x.device)

    def call():
        if lin.ln:
            sq.sq_ln_smooth_quant_act(layer.x, layer.xq, act, layer.g2, layer.b2, 1e-5,
                                      per_tensor_dynamic=True)
        else:
            sq.sq_ln_smooth_quant_act(layer.x, layer.xq, act, inv_s=layer.inv_s,
                                      per_tensor_dynamic=True)

    for _ in range(3):
        call()
    e0 = torch.cuda.Event(enable_timing=True, external=True)
    e1 = torch.cuda.Event(enable_timing=True, external=True)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        e0.record()
        call()
        e1.record()
    times = []
    for i in range(reps):
        flush(i)
        graph.replay()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    sq.sq_sync_status()
    del graph
    ms = statistics.mean(times)
    nbytes = M * K * b + M * K + 4 + (8 * K if lin.ln else 4 * K)
    hbm = load_peaks()[0].get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"shape": f"{M}x{K} {lin.dtype}{' + LayerNorm' if lin.ln else ''}",
            "kernels": "peak pass, step, static quantizer pass (x read twice)",
            "us": round(ms * 1e3, 2), "gbs": round(gbs, 1), "hbm_frac": round(gbs / hbm, 3),
            "bytes": int(nbytes)}


def time_call(torch, call, flush, reps=20):
    """Mean device time (ms) of one call: a CUDA-graph replay per call after
    an L2 flush, device events around it."""
    for _ in range(3):
        call()
    e0 = torch.cuda.Event(enable_timing=True, external=True)
    e1 = torch.cuda.Event(enable_timing=True, external=True)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        e0.record()
        call()
        e1.record()
    times = []
    for i in range(reps):
        flush(i)
        graph.replay()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    del graph
    return statistics.mean(times)


def run_alpha_sweep(sq, torch, layer, lin, flush, alphas=(0.0, 0.25, 0.5, 0.75, 1.0)):
    """alpha chosen by the layer's output error (NEXT-2): the whole smoothed
    layer at five alphas on the step's tokens (eq. (4), fold, quantizer, and
    the GEMM with the fp64 error sums in its epilogue), against the
    unquantized layer in fp32 (the reference is computed once with torch,
    outside the timing)."""
    import torch.nn.functional as F

    xf = layer.x.float()
    if lin.ln:
        xf = F.layer_norm(xf, (lin.K,), layer.gamma, layer.beta, 1e-5)
    y_ref = xf @ layer.w.float().t()
    ws = sq.Workspace(layer.x.device)
    out = {}

    def call():
        out["err"] = sq.sq_alpha_sweep(layer.amax, layer.w, layer.x, y_ref, list(alphas),
                                       layer.gamma, layer.beta, per_token=lin.per_token,
                                       workspace=ws)

    ms = time_call(torch, call, flush, reps=5)
    sq.sq_sync_status()
    err = out["err"].cpu().tolist()
    del y_ref
    return {"shape": f"{lin.T}x{lin.N}x{lin.K}", "alphas": list(alphas),
            "rel_error": [round(e, 6) for e in err], "us_per_alpha": round(ms * 1e3 / len(alphas), 1)}


def run_attention_bmm(sq, torch, dev, flush, heads=32, tokens=2048, head_dim=128):
    """Attention's INT8 matmuls (NEXT-4) at OPT-6.7B shapes, one batched
    launch over the heads each: scores = Q K^T (per-token Q steps, one K step
    per head) and P V (V^T as the K-major operand), bf16 out."""
    g = torch.Generator(device=dev).manual_seed(11)
    peaks, _ = load_peaks()
    int8_peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]) * INT8_PER_BF16
    out = {}
    for name, (M, N, K) in (("scores_qk", (tokens, tokens, head_dim)),
                            ("pv", (tokens, head_dim, tokens))):
        xq = torch.randint(-127, 128, (heads, M, K), dtype=torch.int8, device=dev, generator=g)
        wq = torch.randint(-127, 128, (heads, N, K), dtype=torch.int8, device=dev, generator=g)
        act = torch.rand(heads * M, device=dev, generator=g) * 0.01 + 1e-4
        ws = torch.rand(heads, device=dev, generator=g) * 0.01 + 1e-4
        y = torch.empty((heads, M, N), dtype=torch.bfloat16, device=dev)
        ms = time_call(torch, lambda: sq.sq_bmm_w8a8(xq, wq, act, ws, y, per_token=True,
                                                     w_per_channel=False), flush)
        sq.sq_sync_status()
        tops = 2.0 * heads * M * N * K / (ms * 1e-3) / 1e12
        out[name] = {"shape": f"{heads}x{M}x{N}x{K}", "us": round(ms * 1e3, 2),
                     "tops": round(tops, 1), "int8_frac": round(tops / int8_peak, 3)}
    return out


def run_rms_quant(sq, torch, layer, lin, flush):
    """The quantizer behind an RMSNorm (gamma / s folded, no beta; NEXT-3) on
    the step's activations, per-token; GB/s over x read once + codes and
    scales written once."""
    M, K = lin.T, lin.K
    b = 2 if lin.dtype == "bf16" else 4
    gs = layer.g2 if layer.g2 is not None else layer.inv_s
    act = torch.empty(M, dtype=torch.float32, device=layer.x.device)
    ms = time_call(torch, lambda: sq.sq_rms_smooth_quant_act(layer.x, layer.xq, act, gs),
                   flush)
    sq.sq_sync_status()
    nbytes = M * K * b + M * K + 4 * M + 4 * K
    hbm = load_peaks()[0].get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"shape": f"{M}x{K} {lin.dtype}", "us": round(ms * 1e3, 2), "gbs": round(gbs, 1),
            "hbm_frac": round(gbs / hbm, 3), "bytes": int(nbytes)}


def run_gemm_bias(sq, torch, layer, lin, flush, reps=20):
    """The step's GEMM with the bias epilogue (y = dequantized acc + bias[n]),
    timed like the decode GEMM: one CUDA-graph replay per call after an L2
    flush, device events around it."""
    M, N, K = lin.T, lin.N, lin.K
    g = torch.Generator(device=layer.x.device).manual_seed(7)
    bias = torch.randn(N, device=layer.x.device, generator=g) * 0.1

    def call():
        sq.sq_gemm_w8a8(layer.xq, layer.wq, layer.act, layer.ws, layer.y,
                        per_token=lin.per_token, workspace=layer.workspace, bias=bias)

    for _ in range(3):
        call()
    e0 = torch.cuda.Event(enable_timing=True, external=True)
    e1 = torch.cuda.Event(enable_timing=True, external=True)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        e0.record()
        call()
        e1.record()
    times = []
    for i in range(reps):
        flush(i)
        graph.replay()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    sq.sq_sync_status()
    del graph
    ms = statistics.mean(times)
    peaks, _ = load_peaks()
    int8_peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]) * INT8_PER_BF16
    tops = 2.0 * M * N * K / (ms * 1e-3) / 1e12
    return {"shape": f"{M}x{N}x{K}", "us": round(ms * 1e3, 2), "tops": round(tops, 1),
            "int8_frac": round(tops / int8_peak, 3),
            "note": "one call after an L2 flush, launch included (the step's GEMM share "
                    "overlaps its launch with the quantizer)"}


def run_e2e(sq, torch, layer, lin, d, dev, steps, world, barrier):
    """Same step through the public API, inputs copied from pinned host memory
    every step and the output read back."""
    def pinned(a):
        if a is None:
            return None
        t = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16
             else torch.from_numpy(a))
        return t.pin_memory()

    hx_cal, hx, hw = pinned(d["x_cal"]), pinned(d["x"]), pinned(d["w"])
    hg, hb = pinned(d["gamma"]), pinned(d["beta"])
    hy = torch.empty(layer.y.shape, dtype=layer.y.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hx_cal, hx, hw, hg, hb) if t is not None)
    d2h = hy.numel() * hy.element_size()

    def one():
        layer.x_cal.copy_(hx_cal, non_blocking=True)
        layer.x.copy_(hx, non_blocking=True)
        layer.w.copy_(hw, non_blocking=True)
        if hg is not None:
            layer.gamma.copy_(hg, non_blocking=True)
            layer.beta.copy_(hb, non_blocking=True)
        layer.step()
        hy.copy_(layer.y, non_blocking=True)

    for _ in range(2):
        one()
    barrier()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        one()
    e.record()
    barrier()
    ms = max_over_ranks(s.elapsed_time(e) / steps, world, dev)
    ops = 2.0 * lin.T * lin.N * lin.K
    return {"value": round(throughput_tops(ops, 1, world, ms), 3), "unit": "TOPS",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h)}


# ---------------------------------------------------------------- CPU oracle
def oracle_step_sample(lin, d, frac_tokens, gemm_rows, frac_w):
    """Time the oracle on a bounded sample of each step and extrapolate each
    step linearly in the sampled dimension.  Returns (seconds_full, sample)."""
    import oracle

    oracle.build()
    Tc = max(1, int(lin.T_cal * frac_tokens))
    Tq = max(1, int(lin.T * frac_tokens))
    Nw = max(1, int(lin.N * frac_w))
    t = {}
    t0 = time.perf_counter()
    amax = oracle.calib_absmax(d["x_cal"][:Tc], d["gamma"], d["beta"], 1e-5)
    t["calib"] = (time.perf_counter() - t0) * lin.T_cal / Tc
    t0 = time.perf_counter()
    aw = oracle.weight_colmax(d["w"][:Nw])
    s, inv_s = oracle.smooth_scales(amax, aw, lin.alpha)
    dA = oracle.static_delta(amax, s)
    t["scales"] = (time.perf_counter() - t0) * lin.N / Nw
    t0 = time.perf_counter()
    wq, ws = oracle.fuse_weights_q8(d["w"][:Nw], s)
    if lin.ln:
        g2, b2 = oracle.fold_ln(d["gamma"], d["beta"], s)
    t["fuse"] = (time.perf_counter() - t0) * lin.N / Nw
    t0 = time.perf_counter()
    if lin.ln:
        xq, act, _ = oracle.quant_act(d["x"][:Tq], g2, b2, 1e-5, per_token=lin.per_token,
                                      static_delta=dA)
    else:
        xq, act, _ = oracle.quant_act(d["x"][:Tq], inv_s=inv_s, per_token=lin.per_token,
                                      static_delta=dA)
    t["quant"] = (time.perf_counter() - t0) * lin.T / Tq
    R = max(1, min(gemm_rows, Tq))
    t0 = time.perf_counter()
    oracle.gemm_w8a8(xq[:R], wq, act[:R] if lin.per_token else act, ws,
                     per_token=lin.per_token, out_bf16=(lin.dtype == "bf16"))
    t["gemm"] = (time.perf_counter() - t0) * (lin.T / R) * (lin.N / Nw)
    sample = (f"oracle (single-threaded C) on {Tc}/{lin.T_cal} calibration tokens, "
              f"{Nw}/{lin.N} weight rows, {Tq}/{lin.T} runtime tokens and a {R}x{Nw}x{lin.K} "
              f"GEMM; each step extrapolated linearly to the full workload")
    return sum(t.values()), t, sample


def cpu_baseline(lin, d):
    # the offline steps and the quantizer on every token and weight row, and
    # a quarter of the GEMM's token rows: about 10 s of one host core (the
    # GEMM dominates; the rest is extrapolated from it linearly)
    secs, parts, sample = oracle_step_sample(lin, d, 1, lin.T // 4, 1)
    ops = 2.0 * lin.T * lin.N * lin.K
    return {"value": round(ops / secs / 1e12, 6), "unit": "TOPS", "cores": 1,
            "kind": "oracle", "sample": sample,
            "seconds_per_step_extrapolated": round(secs, 2),
            "parts_s": {k: round(v, 3) for k, v in parts.items()}}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    wl, lin = pick_linear(args)
    d = synth.make_linear_inputs(lin)
    # each step: the oracle on a bounded sample of the step (about 20 ms of
    # one core), extrapolated to the full workload; exactly `steps` of them
    # after at least 3 warm-up samples
    warm = max(3, args.warmup)
    for _ in range(warm):
        oracle_step_sample(lin, d, 1 / 64, 2, 1 / 16)
    secs_all = []
    sample = ""
    for _ in range(max(1, args.steps)):
        secs, _, sample = oracle_step_sample(lin, d, 1 / 64, 2, 1 / 16)
        secs_all.append(secs)
    ops = 2.0 * lin.T * lin.N * lin.K
    total = sum(secs_all)
    value = ops * len(secs_all) / total / 1e12
    line = {
        "metric": METRIC, "value": round(value, 6), "unit": "TOPS", "impl": "reference",
        "n_gpus": world, "steps": len(secs_all), "warmup": warm,
        "ms_per_step": round(total / len(secs_all) * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded outlier-structured activations, random-init weights)",
        "config": config_of(wl, lin, world),
        "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
