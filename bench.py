#!/usr/bin/env python
"""Benchmark of the smoothed W8A8 linear layer (SmoothQuant hot path) on B200.

One step = one pass of the whole path over one batch of synthetic input:
calibration absmax (LayerNorm-fused when a LayerNorm precedes), smoothing
factors (eq. (4)), weight + LayerNorm fold with per-output-channel INT8,
the fused LayerNorm + smoothing + INT8 activation quantizer, and the INT8
tcgen05 GEMM with the dequantizing epilogue.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl reference]

The default workload is the large prefill (calibration peaks over 65536 x
8192 bf16 tokens, then the 8192 -> 28672 linear at 16384 tokens, static
per-tensor activations), the largest single-GPU configuration.
`value` is whole-job throughput in TOPS = 2*M*N*K per step (all ranks) over
the device time of the timed steps, max over ranks.  Each step is one replay
of a CUDA graph of the five calls, timed on the device by event nodes at the
graph's two ends.  The per-call breakdown, taken after the timed steps,
times graphs of the first 1..4 calls the same way: a call's time is what it
adds to the step.  Before every timed replay L2 is flushed outside the timed
events: a 256 MiB buffer is written, then another 256 MiB buffer is read, so
that the timed work finds neither its data nor the flush's dirty lines in
L2.  Inputs are resident in HBM.
`runtime_forward` times what serving pays per batch (the quantizer and the
GEMM) on its own.  `int8_peak` measures the denominator of the GEMM's
roofline on this GPU: the tcgen05 kind::i8 issue rate with no memory traffic
(sq_probe_mma_i8) and cuBLAS's INT8 GEMM at 8192^3 (torch._int_mm).
`e2e` is the same metric through the public Python API with pinned host
buffers: every step copies its inputs host->device and its output back.
`--impl reference` times the CPU oracle (tests-only code) on one host core,
on bounded samples of the same workload, each step extrapolated linearly to
the full workload.
`--profile-call NAME` only runs the named call of the step `--steps` times
after the warm-up steps (for an ncu capture of one kernel) and prints no
line; `--tokens T` and `--cal-tokens T` shrink the runtime and calibration
token counts for such a capture.
"""
from __future__ import annotations

import argparse
import dataclasses
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
DEFAULT_WORKLOAD = "large_prefill_k8192"
SECONDARY_WORKLOAD = "opt6.7b_qkv_t2048"
FLUSH_BYTES = 256 << 20
# nominal ratio of dense int8 to dense bf16 tensor throughput (4.5 : 2.25)
INT8_PER_BF16 = 2.0
SETTLE_S = 3.0  # idle seconds before each secondary measurement
VENDOR_INT8_TOPS = 4500.0  # dense, NVIDIA's figure for B200
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CALLS = ["calib_absmax", "smooth_scales", "fuse_weights_q8", "ln_smooth_quant_act", "gemm_w8a8"]
# DRAM bytes (read + write) of one launch of the step's GEMM, from an ncu
# capture of the current kernel (None until one exists for the workload)
GEMM_DRAM_TRAFFIC = {
    "large_prefill_k8192": (2890703872, "ncu, one launch of gemm_w8a8_tc_kernel<1,256,0,2,4,0,1> "
                            "(CTA pairs) at 16384 x 28672 x 8192: dram__bytes_read.sum 1968.7 MB + "
                            "dram__bytes_write.sum 922.0 MB"),
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
    ap.add_argument("--no-sustained", action="store_true",
                    help="skip the one-second back-to-back GEMM / cuBLAS / probe comparison")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the secondary workload, the HBM rows and the next rows")
    ap.add_argument("--profile-call", default=None, choices=CALLS + ["int8_probe"],
                    help="run only this call (after the warm-up steps) --steps times; no line")
    ap.add_argument("--tokens", type=int, default=None,
                    help="runtime tokens of the workload's linear (profiling of smaller cases)")
    ap.add_argument("--cal-tokens", type=int, default=None,
                    help="calibration tokens of the workload's linear (profiling of smaller cases)")
    return ap.parse_args()


def pick_linear(args, workload=None):
    wl = synth.workloads()[workload or args.workload]
    lin = wl.linears[0]
    if args.linear and workload is None:
        lin = next(l for l in wl.linears if l.name == args.linear)
    if args.tokens and workload is None:
        lin = dataclasses.replace(lin, T=int(args.tokens))
    if args.cal_tokens and workload is None:
        lin = dataclasses.replace(lin, T_cal=int(args.cal_tokens))
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
        self.power = []
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
                self.power.append(self.nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0)
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.005)

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
        out = {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
               "reasons": sorted(self.reasons), "samples": len(self.samples)}
        if self.power:
            out["power_w_median"] = round(statistics.median(self.power), 1)
        return out


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
        # per-token steps are written by the quantizer; a static step is the
        # one the smoothing call derives (dA), read by the quantizer and GEMM
        self.act = torch.empty(M, dtype=f32, device=dev) if lin.per_token else self.dA
        self.y = torch.empty((M, N), dtype=io, device=dev)
        self.workspace = sq.Workspace(dev)
        # this library's kernels per step: calibration peak; column peak +
        # eq. (4) factors; weight fold (which also divides gamma and beta by
        # s); quantizer; GEMM
        self.kernels_per_step = 6

    def step(self, ev=None, upto=5, start=1):
        """Calls start..upto of the five (1..5: one step); ev = (start, end)
        events recorded around them, or None.  (Running the weight column
        peaks on a second stream beside the calibration was measured no
        faster: whichever kernel starts first fills the SMs.)"""
        sq, L = self.sq, self.lin
        if ev is not None:
            ev[0].record()
        if start <= 1 <= upto:
            self.amax.zero_()
            sq.sq_calib_absmax(self.x_cal, self.amax, self.gamma, self.beta, 1e-5)
        if start <= 2 <= upto:
            sq.sq_smooth_scales(self.amax, self.w, L.alpha, self.s, self.inv_s,
                                None if L.per_token else self.dA)
        if start <= 3 <= upto:
            sq.sq_fuse_weights_q8(self.w, self.s, self.wq, self.ws, self.gamma, self.beta,
                                  self.g2, self.b2)
        if start <= 4 <= upto:
            if L.ln:
                sq.sq_ln_smooth_quant_act(self.x, self.xq, self.act, self.g2, self.b2, 1e-5,
                                          per_token=L.per_token)
            else:
                sq.sq_ln_smooth_quant_act(self.x, self.xq, self.act, inv_s=self.inv_s,
                                          per_token=L.per_token)
        if start <= 5 <= upto:
            sq.sq_gemm_w8a8(self.xq, self.wq, self.act, self.ws, self.y, per_token=L.per_token,
                            workspace=self.workspace)
        if ev is not None:
            ev[1].record()

    def call(self, name):
        """One of the five calls on its own (inputs from an earlier step)."""
        j = CALLS.index(name) + 1
        self.step(upto=j, start=j)


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


def time_step_graphs(torch, layer, flush, K, clocks=None, prefixes=True):
    """Step times (ms) of K replays of the whole step's graph, each after an
    L2 flush, device events at the graph's two ends; then (prefixes) the
    mean time of graphs of the first 1..4 calls, so that a call's time is
    what it adds to the step."""

    def capture(upto, start=1):
        ev = (torch.cuda.Event(enable_timing=True, external=True),
              torch.cuda.Event(enable_timing=True, external=True))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            layer.step(ev, upto, start)
        return g, ev

    def replay(g, ev, n):
        t = []
        for i in range(n):
            flush(i)  # evicts the previous replay's data from L2
            g.replay()
            torch.cuda.synchronize()
            t.append(ev[0].elapsed_time(ev[1]))
        return t

    graph, ev_step = capture(5)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    if clocks is not None:
        with clocks:
            step_ms = replay(graph, ev_step, K)
    else:
        step_ms = replay(graph, ev_step, K)
    del graph
    if not prefixes:
        return step_ms, None
    prefix_ms = {0: 0.0, 5: statistics.mean(step_ms)}
    for upto in range(1, 5):
        g, ev = capture(upto)
        g.replay()
        prefix_ms[upto] = statistics.mean(replay(g, ev, K))
        del g
    per = {n: prefix_ms[j + 1] - prefix_ms[j] for j, n in enumerate(CALLS)}
    return step_ms, per


def kernel_table(lin, per, hbm, int8_peak):
    ops = 2.0 * lin.T * lin.N * lin.K
    ab = algorithmic_bytes(lin)
    kernels = {}
    for n in CALLS:
        ms = per[n]
        k = {"ms": round(ms, 5), "bytes": int(ab[n]),
             "gbs": round(ab[n] / (ms * 1e-3) / 1e9, 1),
             "hbm_frac": round(ab[n] / (ms * 1e-3) / 1e9 / hbm, 3)}
        if n == "gemm_w8a8":
            tops = ops / (ms * 1e-3) / 1e12
            k["tops"] = round(tops, 1)
            k["int8_frac"] = round(tops / int8_peak, 3)
            k["int8_frac_vendor"] = round(tops / VENDOR_INT8_TOPS, 3)
        kernels[n] = k
    return kernels


def measure_int8_peak(sq, torch, dev, clocks_cls):
    """The dense INT8 tensor-core ceiling of this GPU, measured two ways:
    (1) the tcgen05.mma kind::i8 issue rate with the operands in shared
    memory and no other work, one CTA per SM (sq_probe_mma_i8) and on CTA
    pairs (sq_probe_mma_i8_pair, the GEMM's instruction form), in bursts of
    about 2 ms with idle gaps -- the way the step's GEMM runs in the timed
    region -- and, for context, back to back for ~30 ms launches, where the
    power cap lowers the clock; (2) cuBLAS's INT8 GEMM (torch._int_mm) at
    8192^3.  Best of several launches each, CUDA events on the launching
    stream, NVML clock sampled during each.  The largest of the burst probes
    and cuBLAS is the roofline's peak."""
    sms = torch.cuda.get_device_properties(dev).multi_processor_count

    def ev_time(fn, reps, warm, gap_s=0.0):
        for _ in range(warm):
            fn()
        torch.cuda.synchronize()
        best = None
        for _ in range(reps):
            if gap_s:
                time.sleep(gap_s)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            t = e0.elapsed_time(e1)
            best = t if best is None else min(best, t)
        return best

    out = {}
    pairs = sms // 2
    for name, kblocks, reps, gap, pair in (
            ("tcgen05_i8_probe", 8000, 10, 0.05, False),
            ("tcgen05_i8_pair_probe", 8000, 10, 0.05, True),
            ("tcgen05_i8_probe_sustained", 100_000, 5, 0.0, False)):
        clocks = clocks_cls(torch.cuda.current_device())
        if pair:
            fn = lambda: sq.sq_probe_mma_i8_pair(kblocks, pairs)  # noqa: E731
            ops = 16777216.0 * kblocks * pairs
            mma = "256x256x32 kind::i8 on CTA pairs (cta_group::2), operands in smem"
        else:
            fn = lambda: sq.sq_probe_mma_i8(kblocks, sms)  # noqa: E731
            ops = 8388608.0 * kblocks * sms
            mma = "128x256x32 kind::i8, one accumulator, operands in smem"
        with clocks:
            ms = ev_time(fn, reps, 2, gap)
        st = sq.sq_sync_status()
        tops = ops / (ms * 1e-3) / 1e12
        out[name] = {"tops": round(tops, 1), "ms": round(ms, 3), "ctas": sms,
                     "kblocks_per_cta": kblocks, "idle_gap_s": gap, "mma": mma,
                     "clocks": clocks.summary(), "status": st}
    probe_tops = max(out["tcgen05_i8_probe"]["tops"], out["tcgen05_i8_pair_probe"]["tops"])
    probe_name = ("tcgen05_i8_pair_probe" if out["tcgen05_i8_pair_probe"]["tops"] >=
                  out["tcgen05_i8_probe"]["tops"] else "tcgen05_i8_probe")
    n = 8192
    g = torch.Generator(device=dev).manual_seed(5)
    a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev, generator=g)
    b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev, generator=g)
    try:
        ms2 = ev_time(lambda: torch._int_mm(a, b.t()), 10, 3)
        cub = 2.0 * n ** 3 / (ms2 * 1e-3) / 1e12
        out["cublas_int8_gemm_8192"] = {"tops": round(cub, 1), "ms": round(ms2, 3),
                                        "call": "torch._int_mm (cuBLASLt), int32 out"}
    except Exception as e:  # noqa: BLE001 - reported, the probe still stands
        cub = 0.0
        out["cublas_int8_gemm_8192"] = {"error": str(e)[:200]}
    del a, b
    out["peak_tops"] = round(max(probe_tops, cub), 1)
    out["peak_from"] = probe_name if probe_tops >= cub else "cublas_int8_gemm_8192"
    out["vendor_dense_tops"] = VENDOR_INT8_TOPS
    return out


def profile_only(args, sq, torch, layer, flush):
    """--profile-call: the named call alone, --steps times, nothing printed."""
    for _ in range(max(1, args.warmup)):
        layer.step()
    torch.cuda.synchronize()
    for i in range(args.steps):
        if args.profile_call == "int8_probe":
            sq.sq_probe_mma_i8_pair(2000, torch.cuda.get_device_properties(0).multi_processor_count // 2)
            sq.sq_probe_mma_i8(2000, torch.cuda.get_device_properties(0).multi_processor_count)
        else:
            layer.call(args.profile_call)
    torch.cuda.synchronize()
    sq.sq_sync_status()


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
    if args.profile_call:
        profile_only(args, sq, torch, layer, flush)
        return

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    warm = max(3, args.warmup)
    for _ in range(warm):
        layer.step()
    sq.sq_sync_status()

    # the timed region: K replays of the step's graph (five calls, six
    # kernels), event nodes only at its two ends
    K = args.steps
    clocks = ClockSampler(torch.cuda.current_device())
    barrier()
    step_ms, per = time_step_graphs(torch, layer, flush, K, clocks)
    barrier()
    sq.sq_sync_status()
    total_ms = max_over_ranks(float(sum(step_ms)), world, dev)
    ops = 2.0 * lin.T * lin.N * lin.K
    value = throughput_tops(ops, K, world, total_ms)

    peaks, peak_kind = load_peaks()
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    bf16_peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    int8 = measure_int8_peak(sq, torch, dev, ClockSampler)
    int8_peak = int8["peak_tops"]
    kernels = kernel_table(lin, per, hbm, int8_peak)
    gemm_tops = kernels["gemm_w8a8"]["tops"]

    def settled(fn):
        """fn() after SETTLE_S seconds of an idle GPU, with the SM clock
        sampled while it runs (added to a dict result as "clocks").  Right
        after a long burst (the INT8 probes, the step loops) the SM clock was
        seen at about 1540 MHz for a few seconds, no throttle reason set, and
        a short kernel timed then read up to 30 % slow."""
        torch.cuda.synchronize()
        time.sleep(SETTLE_S)
        cs = ClockSampler(torch.cuda.current_device())
        with cs:
            r = fn()
        return {**r, "clocks": cs.summary()} if isinstance(r, dict) else r

    # what serving pays per batch: the quantizer and the GEMM alone
    def forward():
        fwd_ms = time_graph_calls(torch, lambda: layer.step(upto=5, start=4), flush, K)
        return {
            "calls": "sq_ln_smooth_quant_act + sq_gemm_w8a8 (the offline steps excluded)",
            "us": round(fwd_ms * 1e3, 2), "tops": round(ops / (fwd_ms * 1e-3) / 1e12, 1),
            "int8_frac": round(ops / (fwd_ms * 1e-3) / 1e12 / int8_peak, 3)}

    runtime_forward = settled(forward)

    # ---- e2e through the public API with pinned host buffers
    e2e = run_e2e(sq, torch, layer, lin, d, dev, args.e2e_steps, world, barrier)
    small_m = None if args.no_small_m else settled(lambda: run_small_m(sq, torch, dev, flush))
    extras = {}
    if not args.no_extras:
        extras["secondary_workloads"] = {
            SECONDARY_WORKLOAD: settled(
                lambda: run_secondary(args, sq, torch, dev, flush, hbm, int8_peak))}
        extras["hbm_rows"] = settled(lambda: run_hbm_rows(sq, torch, dev, flush, hbm))
        extras["gemm_13b_layer"] = settled(lambda: run_13b_gemms(sq, torch, dev, flush, int8_peak))
        extras["next_rows"] = {
            "o2_per_tensor_dynamic_quant": settled(lambda: run_o2(sq, torch, layer, lin, flush)),
            "gemm_bias_epilogue": settled(
                lambda: run_gemm_bias(sq, torch, layer, lin, flush, int8_peak)),
            "rmsnorm_quant_per_token": settled(lambda: run_rms_quant(sq, torch, layer, lin, flush)),
            "alpha_sweep": settled(lambda: run_alpha_sweep(sq, torch, layer, lin, flush)),
            "attention_bmm": settled(
                lambda: run_attention_bmm(sq, torch, layer.x.device, flush, int8_peak))}
    if not args.no_extras and not args.no_sustained:
        extras["sustained_power_cap"] = run_sustained(sq, torch, layer, lin)

    traffic = GEMM_DRAM_TRAFFIC.get(wl.name, (None, None))
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": K,
        "warmup": warm,
        "ms_per_step": round(total_ms / K, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8",
        "data": "synthetic (seeded outlier-structured activations, random-init weights)",
        "config": config_of(wl, lin, world),
        "roofline": {
            "bound": "tensor",
            "kernel": "gemm_w8a8 (tcgen05.mma kind::i8), its share of the step",
            "achieved": round(gemm_tops, 1),
            "peak": int8_peak,
            "unit": "TFLOP/s",
            "frac": round(gemm_tops / int8_peak, 4),
            "frac_vendor": round(gemm_tops / VENDOR_INT8_TOPS, 4),
            "frac_bf16x2": round(gemm_tops / (bf16_peak * INT8_PER_BF16), 4),
            "traffic": traffic[0],
            "traffic_source": traffic[1],
            "peak_note": f"int8 ops; peak measured live on this GPU ({int8['peak_from']}); "
                         f"frac_vendor against the dense {VENDOR_INT8_TOPS:.0f} TOPS spec; "
                         f"frac_bf16x2 against the {peak_kind} bf16 burst {bf16_peak} TFLOP/s x 2",
        },
        "int8_peak": int8,
        "kernels": kernels,
        "runtime_forward": runtime_forward,
        "small_m_decode": small_m,
        **extras,
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


def time_graph_calls(torch, fn, flush, reps):
    """Mean device time (ms) of fn captured as one CUDA graph, replayed reps
    times, each replay after an L2 flush, device events at its two ends."""
    e0 = torch.cuda.Event(enable_timing=True, external=True)
    e1 = torch.cuda.Event(enable_timing=True, external=True)
    fn()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        e0.record()
        fn()
        e1.record()
    graph.replay()
    t = []
    for i in range(reps):
        flush(i)
        graph.replay()
        torch.cuda.synchronize()
        t.append(e0.elapsed_time(e1))
    del graph
    return statistics.mean(t)


def run_sustained(sq, torch, layer, lin, seconds=1.0):
    """The step's GEMM, cuBLAS's INT8 GEMM on the same operands (torch._int_mm,
    int32 out) and the tcgen05 probe, each back to back for about `seconds`
    so that the board's power cap engages, with the SM clock and the board
    power sampled.  int8 ops per clock per SM compares the three at whatever
    clock the cap leaves each; the tensor cores' ceiling is 16384 (8192
    multiply-adds per clock per SM)."""
    sms = torch.cuda.get_device_properties(layer.x.device).multi_processor_count
    ops = 2.0 * lin.T * lin.N * lin.K
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        layer.call("gemm_w8a8")
    xq, wq = layer.xq, layer.wq
    entries = (("gemm_w8a8", lambda: graph.replay(), ops),
               ("cublas_int_mm_same_shape", lambda: torch._int_mm(xq, wq.t()), ops),
               ("tcgen05_i8_probe", lambda: sq.sq_probe_mma_i8(8000, sms), 8388608.0 * 8000 * sms))
    out = {}
    for name, fn, n_ops in entries:
        try:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            fn()  # the first call may allocate or initialise a library
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            n = max(20, int(seconds * 1e3 / e0.elapsed_time(e1)))
            time.sleep(SETTLE_S)
            cs = ClockSampler(torch.cuda.current_device())
            with cs:
                e0.record()
                for _ in range(n):
                    fn()
                e1.record()
                torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / n
            tops = n_ops / (ms * 1e-3) / 1e12
            c = cs.summary()
            per_clk = (round(tops * 1e12 / (c["sm_mhz"] * 1e6 * sms))
                       if c.get("sm_mhz") else None)
            out[name] = {"launches": n, "ms_per_launch": round(ms, 4), "tops": round(tops, 1),
                         "int8_ops_per_clock_per_sm": per_clk, "clocks": c}
        except Exception as e:  # noqa: BLE001 - reported; the rest still stands
            out[name] = {"error": str(e)[:200]}
    del graph
    sq.sq_sync_status()
    return out


def run_secondary(args, sq, torch, dev, flush, hbm, int8_peak):
    """The OPT-6.7B-shaped QKV step (LayerNorm, per-token) timed like the
    headline step: whole-step TOPS and the per-call breakdown."""
    _, lin = pick_linear(args, SECONDARY_WORKLOAD)
    d = synth.make_linear_inputs(lin)
    layer = Layer(sq, torch, lin, d, dev)
    for _ in range(3):
        layer.step()
    step_ms, per = time_step_graphs(torch, layer, flush, max(args.steps, 20))
    sq.sq_sync_status()
    ms = statistics.mean(step_ms)
    ops = 2.0 * lin.T * lin.N * lin.K
    fwd_ms = time_graph_calls(torch, lambda: layer.step(upto=5, start=4), flush, 20)
    out = {"config": config_of(synth.workloads()[SECONDARY_WORKLOAD], lin, 1),
           "ms_per_step": round(ms, 5), "tops": round(ops / (ms * 1e-3) / 1e12, 1),
           "kernels": kernel_table(lin, per, hbm, int8_peak),
           "runtime_forward": {"us": round(fwd_ms * 1e3, 2),
                               "tops": round(ops / (fwd_ms * 1e-3) / 1e12, 1)}}
    del layer
    return out


def run_hbm_rows(sq, torch, dev, flush, hbm):
    """HBM-bound steps at sizes where they are HBM-bound (inputs far larger
    than L2): the 13B fc2 input quantizer (4096 x 20480 bf16, per-token,
    x * 1/s) and its raw calibration peak, each one graph replay after an
    L2 flush."""
    lin = next(l for l in synth.workloads()["13b_layer_t4096"].linears if l.name == "fc2_a0.5")
    K, T = lin.K, lin.T
    out_ch = synth.outlier_pattern(lin.seed, K, lin.outlier_frac, tag=f"k{K}")
    x = torch.from_numpy(synth.bf16_bits(synth.activations(
        lin.seed, "bench/fc2_x", T, K, out_ch, relu=True)).view(np.int16)).view(torch.bfloat16).to(dev)
    g = torch.Generator(device=dev).manual_seed(17)
    inv_s = torch.rand(K, device=dev, generator=g) * 1.9 + 0.02
    xq = torch.empty((T, K), dtype=torch.int8, device=dev)
    act = torch.empty(T, dtype=torch.float32, device=dev)
    amax = torch.zeros(K, dtype=torch.float32, device=dev)
    res = {}
    ms = time_graph_calls(torch, lambda: sq.sq_ln_smooth_quant_act(x, xq, act, inv_s=inv_s,
                                                                   per_token=True), flush, 20)
    nb = T * K * 2 + T * K + 4 * T + 4 * K
    res["13b_fc2_quant_per_token"] = {"shape": f"{T}x{K} bf16, x * 1/s", "us": round(ms * 1e3, 2),
                                      "bytes": nb, "gbs": round(nb / (ms * 1e-3) / 1e9, 1),
                                      "hbm_frac": round(nb / (ms * 1e-3) / 1e9 / hbm, 3)}
    ms = time_graph_calls(torch, lambda: sq.sq_calib_absmax(x, amax), flush, 20)
    nb = T * K * 2 + 4 * K
    res["13b_fc2_calib_absmax"] = {"shape": f"{T}x{K} bf16, raw", "us": round(ms * 1e3, 2),
                                   "bytes": nb, "gbs": round(nb / (ms * 1e-3) / 1e9, 1),
                                   "hbm_frac": round(nb / (ms * 1e-3) / 1e9 / hbm, 3)}
    sq.sq_sync_status()
    return res


def run_13b_gemms(sq, torch, dev, flush, int8_peak):
    """The four GEMMs of the 13B layer (4096 tokens, hidden 5120: QKV, out,
    fc1, fc2), per-token steps, bf16 out, each one CUDA-graph replay after an
    L2 flush; TOPS against the measured INT8 peak."""
    g = torch.Generator(device=dev).manual_seed(23)
    out = {}
    for lin in synth.workloads()["13b_layer_t4096"].linears:
        if not lin.name.endswith("_a0.5"):
            continue
        M, N, K = lin.T, lin.N, lin.K
        xq = torch.randint(-127, 128, (M, K), dtype=torch.int8, device=dev, generator=g)
        wq = torch.randint(-127, 128, (N, K), dtype=torch.int8, device=dev, generator=g)
        act = torch.rand(M, device=dev, generator=g) * 0.01 + 1e-4
        ws = torch.rand(N, device=dev, generator=g) * 0.01 + 1e-4
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        wsp = sq.Workspace(dev)
        ms = time_call(torch, lambda: sq.sq_gemm_w8a8(xq, wq, act, ws, y, per_token=True,
                                                     workspace=wsp), flush)
        tops = 2.0 * M * N * K / (ms * 1e-3) / 1e12
        out[lin.name.split("_")[0]] = {"shape": f"{M}x{N}x{K}", "us": round(ms * 1e3, 2),
                                       "tops": round(tops, 1), "int8_frac": round(tops / int8_peak, 3)}
        del xq, wq, y
    sq.sq_sync_status()
    return out


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


def run_attention_bmm(sq, torch, dev, flush, int8_peak, heads=32, tokens=2048, head_dim=128):
    """Attention's INT8 matmuls (NEXT-4) at OPT-6.7B shapes, one batched
    launch over the heads each: scores = Q K^T (per-token Q steps, one K step
    per head) and P V (V^T as the K-major operand), bf16 out."""
    g = torch.Generator(device=dev).manual_seed(11)
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


def run_gemm_bias(sq, torch, layer, lin, flush, int8_peak, reps=20):
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
    tops = 2.0 * M * N * K / (ms * 1e-3) / 1e12
    return {"shape": f"{M}x{N}x{K}", "us": round(ms * 1e3, 2), "tops": round(tops, 1),
            "int8_frac": round(tops / int8_peak, 3),
            "note": "one call after an L2 flush, launch included (the step's GEMM share "
                    "overlaps its launch with the quantizer)"}


def run_e2e(sq, torch, layer, lin, d, dev, steps, world, barrier):
    """The same step through the public API, every step uploading all of its
    inputs from pinned host memory and reading its whole output back, run
    the way a serving loop would: two sets of device buffers, the uploads on
    one copy stream and the read-backs on another, so that step i's output
    travels to the host while step i+1's inputs travel to the device (PCIe
    moves both directions at once) and the kernels run in between.  Events
    order each buffer's reuse: an upload waits until the step that last used
    its buffers has computed, a step waits for its upload and for the
    read-back of the output it will overwrite."""
    def pinned(a):
        if a is None:
            return None
        t = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16
             else torch.from_numpy(a))
        return t.pin_memory()

    hx_cal, hx, hw = pinned(d["x_cal"]), pinned(d["x"]), pinned(d["w"])
    hg, hb = pinned(d["gamma"]), pinned(d["beta"])
    layers = [layer, Layer(sq, torch, lin, d, dev)]
    hy = [torch.empty(layer.y.shape, dtype=layer.y.dtype).pin_memory() for _ in layers]
    h2d = sum(t.numel() * t.element_size() for t in (hx_cal, hx, hw, hg, hb) if t is not None)
    d2h = hy[0].numel() * hy[0].element_size()
    s_comp = torch.cuda.current_stream()
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    computed = [torch.cuda.Event() for _ in layers]
    uploaded = [torch.cuda.Event() for _ in layers]
    read_back = [torch.cuda.Event() for _ in layers]

    def one(i):
        k = i % 2
        L = layers[k]
        with torch.cuda.stream(s_up):
            s_up.wait_event(computed[k])  # the step that last read these inputs is done
            L.x_cal.copy_(hx_cal, non_blocking=True)
            L.x.copy_(hx, non_blocking=True)
            L.w.copy_(hw, non_blocking=True)
            if hg is not None:
                L.gamma.copy_(hg, non_blocking=True)
                L.beta.copy_(hb, non_blocking=True)
            uploaded[k].record(s_up)
        s_comp.wait_event(uploaded[k])
        s_comp.wait_event(read_back[k])  # the output this step overwrites is on the host
        L.step()
        computed[k].record(s_comp)
        with torch.cuda.stream(s_down):
            s_down.wait_event(computed[k])
            hy[k].copy_(L.y, non_blocking=True)
            read_back[k].record(s_down)

    for i in range(2):
        one(i)
    barrier()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(s_up)
    for i in range(steps):
        one(i)
    e.record(s_down)
    barrier()
    ms = max_over_ranks(s.elapsed_time(e) / steps, world, dev)
    ops = 2.0 * lin.T * lin.N * lin.K
    del layers[1]
    return {"value": round(throughput_tops(ops, 1, world, ms), 3), "unit": "TOPS",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h),
            "pipelining": "two device buffer sets; uploads, kernels and read-backs on three "
                          "streams, step i's read-back beside step i+1's upload"}


# ---------------------------------------------------------------- CPU oracle
def host_record():
    """The host the oracle runs on: CPU model, logical CPUs, and the core
    the timing thread is pinned to."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count()}


class PinnedToOneCore:
    """Pins the calling thread to one allowed core (the highest-numbered,
    away from the usual interrupt and driver cores) for the oracle timing,
    and restores the previous affinity afterwards."""

    def __enter__(self):
        self.prev = os.sched_getaffinity(0)
        self.core = max(self.prev)
        os.sched_setaffinity(0, {self.core})
        return self

    def __exit__(self, *a):
        os.sched_setaffinity(0, self.prev)


def oracle_step_sample(lin, d, Tc, Tq, Nw, R):
    """Time the oracle on a bounded sample of each step -- the first Tc
    calibration tokens, Nw weight rows, Tq runtime tokens and an R x Nw x K
    GEMM of `d` -- and extrapolate each step linearly in the sampled
    dimension to lin's full sizes.  Returns (seconds_full, parts, sample)."""
    import oracle

    oracle.build()
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
    R = max(1, min(R, Tq))
    t0 = time.perf_counter()
    oracle.gemm_w8a8(xq[:R], wq, act[:R] if lin.per_token else act, ws,
                     per_token=lin.per_token, out_bf16=(lin.dtype == "bf16"))
    t["gemm"] = (time.perf_counter() - t0) * (lin.T / R) * (lin.N / Nw)
    sample = (f"oracle (single-threaded C, one pinned core) on {Tc}/{lin.T_cal} calibration "
              f"tokens, {Nw}/{lin.N} weight rows, {Tq}/{lin.T} runtime tokens and a "
              f"{R}x{Nw}x{lin.K} GEMM; each step extrapolated linearly to the full workload")
    return sum(t.values()), t, sample


def cpu_baseline(lin, d):
    # the offline steps and the quantizer on every token and weight row, and
    # 48 of the GEMM's token rows (one host core, about 15 s; the GEMM is
    # extrapolated from them linearly)
    with PinnedToOneCore() as pin:
        t0 = time.perf_counter()
        secs, parts, sample = oracle_step_sample(lin, d, lin.T_cal, lin.T, lin.N, 48)
        timed = time.perf_counter() - t0
    ops = 2.0 * lin.T * lin.N * lin.K
    return {"value": round(ops / secs / 1e12, 6), "unit": "TOPS", "cores": 1,
            "kind": "oracle", "sample": sample, "extrapolated": True,
            "seconds_per_step_extrapolated": round(secs, 2),
            "seconds_timed": round(timed, 2), "pinned_core": pin.core, **host_record(),
            "parts_s": {k: round(v, 3) for k, v in parts.items()}}


# the reference arm's sample: 1/16 of the tokens, 1/8 of the weight rows and
# a 2-row GEMM of the workload, drawn with the workload's own recipe (about
# half a second of one host core per step at the large prefill)
REF_FRAC_TOKENS, REF_FRAC_W, REF_GEMM_ROWS = 16, 8, 2


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    wl, lin = pick_linear(args)
    Tc = max(1, lin.T_cal // REF_FRAC_TOKENS)
    Tq = max(1, lin.T // REF_FRAC_TOKENS)
    Nw = max(1, lin.N // REF_FRAC_W)
    d = synth.make_linear_inputs(lin, T=Tq, T_cal=Tc, N=Nw)
    # each step: the oracle on the bounded sample, extrapolated to the full
    # workload; exactly `steps` of them after at least 3 warm-up samples
    warm = max(3, args.warmup)
    secs_all, timed_all = [], []
    sample = ""
    with PinnedToOneCore() as pin:
        for _ in range(warm):
            oracle_step_sample(lin, d, Tc, Tq, Nw, REF_GEMM_ROWS)
        for _ in range(max(1, args.steps)):
            t0 = time.perf_counter()
            secs, _, sample = oracle_step_sample(lin, d, Tc, Tq, Nw, REF_GEMM_ROWS)
            timed_all.append(time.perf_counter() - t0)
            secs_all.append(secs)
    ops = 2.0 * lin.T * lin.N * lin.K
    total = sum(secs_all)
    value = ops * len(secs_all) / total / 1e12
    line = {
        "metric": METRIC, "value": round(value, 6), "unit": "TOPS", "impl": "reference",
        "n_gpus": world, "steps": len(secs_all), "warmup": warm,
        "ms_per_step": round(total / len(secs_all) * 1e3, 3),
        "ms_per_step_is": "extrapolated from the timed sample to the full workload",
        "sample_ms_per_step": round(sum(timed_all) / len(timed_all) * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded outlier-structured activations, random-init weights)",
        "config": config_of(wl, lin, world),
        "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": 1, "kind": "oracle",
                         "sample": sample, "extrapolated": True, "pinned_core": pin.core,
                         **host_record()},
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
