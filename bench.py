#!/usr/bin/env python3
"""Benchmark of the FP32 NCHW conv2d forward library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload depthwise|tiny_grouped|fused_chain|dense_5x9]
                    [--no-shapes] [--force-kernel NAME]
    python bench.py --profile --workload NAME [--batch B] [--calls C]   (ncu target)

One step = one call of the library's entry point on one batch of the
workload (default: the depthwise conv of a MobileNetV2 inverted-residual
block, x[4,144,56,56], 3x3, s1, p1, groups=144).  Metric: algorithmic GB/s
(x read once + w read once + y written once, per second), with GFLOP/s
(2 x multiply-accumulates) and the roofline fraction alongside.

Timing boundaries (the "GroupConv Atlas" distinguishes both):
  value      device events around a CUDA graph holding exactly K captured
             calls; inputs stay resident in HBM; consecutive calls rotate
             through a pool of input/output buffers larger than 4 x L2, so no
             call finds its data in L2.  The two events are record nodes
             inside the graph: the first on a side branch after one untimed
             lead-in call, the second after the K-th call, so the interval
             holds exactly K calls in steady state and neither the graph's
             launch nor the first call's unoverlapped launch latency.
  e2e        per step: pinned-host -> device copy of the inputs, the call,
             device -> pinned-host copy of the output, timed with events on
             the same stream.
  sync_api   host clock around one eager call + stream synchronize
             (median over K calls).
The oracle (FP64 CPU loop nest) is timed on the host cores as a reported
baseline (`cpu_baseline`), and is what `--impl reference` times.

Multi-GPU: every rank runs its own batch (the work shards along N with no
exchange), time = max over ranks, value = all ranks' bytes / that time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from depthwise_convolution_fp32_b200 import inputs  # noqa: E402
from depthwise_convolution_fp32_b200 import workloads as wl  # noqa: E402

METRIC = "conv2d FP32 GB/s + GFLOP/s per shape, fraction of roofline (graph & sync timing)"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
PROFILES = os.path.join(ROOT, "profiles")


# ------------------------------------------------------------------ helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured", d
    except Exception:
        return FALLBACK_HBM_GBS, "fallback", {}


KERNEL_TU = {"depthwise": "direct_conv.cu", "tiny_grouped": "direct_conv.cu",
             "dense_5x9": "igemm_tf32.cu", "fused_chain": "igemm_tf32.cu"}


def kernel_source_hash(tu: str) -> str:
    """Hash of one kernel translation unit and the headers every kernel
    includes; a stored ncu traffic figure is only valid for the sources it
    was captured from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "depthwise_convolution_fp32_b200", "csrc")
    for f in (tu, "device_utils.cuh", "gconv_internal.h"):
        h.update(f.encode())
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def stored_traffic(workload: str):
    """DRAM bytes per launch of the dominant kernel from a committed ncu
    summary, or None when absent or captured from different sources."""
    path = os.path.join(PROFILES, "traffic.json")
    try:
        d = json.load(open(path))
        e = d[workload]
        if e.get("source_hash") != kernel_source_hash(KERNEL_TU[workload]):
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


def max_over_ranks(values, device, world):
    """Element-wise maximum of per-rank timings (the job takes as long as its
    slowest rank); identity on one rank."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def weak_scaling_rate(units_per_step, world, steps, ms):
    """Whole-job rate: every rank processes `units_per_step` per step."""
    return units_per_step * world * steps / (ms / 1e3)


TF32_OVER_BF16 = 1.1 / 2.25      # nominal dense tf32 / bf16 tensor throughput on B200

# Compute rates measured on this GPU at start-up by libgconv_peaks.so (FP32
# FMA; tcgen05 kind::tf32 and kind::f16/bf16 MMA), reported beside the roofline
# denominators to corroborate them.
MEASURED_COMPUTE = {}


def measure_compute_peaks():
    """FP32 CUDA-core and tensor-core MMA rates of this GPU (TFLOP/s), each
    from one timed launch of a throughput microbenchmark (a few ms each)."""
    import ctypes
    from depthwise_convolution_fp32_b200 import build
    lib = ctypes.CDLL(build.build_peaks())
    out = {}
    for name, fn, iters in (("fp32_fma", lib.gpeaks_ffma, 4096), ("tf32_mma", lib.gpeaks_mma_tf32, 20000),
                            ("bf16_mma", lib.gpeaks_mma_bf16, 20000)):
        fn.restype = ctypes.c_int
        fn.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]
        ms, fl = ctypes.c_double(0), ctypes.c_double(0)
        rc = fn(iters, ctypes.byref(ms), ctypes.byref(fl))
        if rc == 0 and ms.value > 0:
            out[name + "_tflops"] = round(fl.value / (ms.value * 1e-3) / 1e12, 2)
            out[name + "_ms"] = round(ms.value, 3)
    if "tf32_mma_tflops" in out and "bf16_mma_tflops" in out:
        # one useful FP32-accurate multiply-add = one tf32 MAC + two bf16 MACs
        t, b = out["tf32_mma_tflops"], out["bf16_mma_tflops"]
        out["fp32_accurate_tensor_tflops"] = round(1.0 / (1.0 / t + 2.0 / b), 2)
    MEASURED_COMPUTE.update(out)
    return out


def fp32_peak_tflops():
    """Roofline denominator of the CUDA-core path (bound "alu"): 148 SMs x 128
    FP32 FMA lanes x 2 FLOP x 1965 MHz, from unit counts and the clock.  The
    FMA microbenchmark's measured rate is reported beside it (compute_peaks)."""
    return wl.fp32_fma_peak_tflops()


def tensor_fp32_peak_tflops(meas):
    """Roofline denominator of the tensor-core path: useful FP32 FLOP/s when
    each multiply-add costs one tf32 MAC (main term) plus two bf16 MACs (the
    two cross terms, one K=16 bf16 MMA per 8 channels).  With the measured bf16
    GEMM peak (MEASURED_PEAKS.json, else the 1.59 PFLOP/s fallback) and the
    nominal tf32/bf16 ratio r: bf16 / (1/r + 2).  The tcgen05 MMA
    microbenchmarks' tf32 and bf16 rates are reported beside it."""
    bf16 = float(meas.get("bf16_tflops", 1590.0)) if meas else 1590.0
    return bf16 / (1.0 / TF32_OVER_BF16 + 2.0)


def roofline_for(wk, sec, plan, hbm_peak, meas):
    """Binding roofline term of one call: HBM bytes, FP32 CUDA-core FLOPs or
    the tensor-core FP32-accurate ceiling (for the implicit-GEMM plan)."""
    t_hbm = wk.bytes / (hbm_peak * 1e9)
    if plan.startswith("igemm"):
        peak_c = tensor_fp32_peak_tflops(meas)
        bound_c = "tensor"
    else:
        peak_c = fp32_peak_tflops()
        bound_c = "alu"
    t_cmp = wk.flops / (peak_c * 1e12)
    if t_hbm >= t_cmp:
        ach = wk.bytes / sec / 1e9
        return {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(ach / hbm_peak, 4)}
    ach = wk.flops / sec / 1e12
    return {"bound": bound_c, "achieved": round(ach, 2), "peak": round(peak_c, 1), "unit": "TFLOP/s",
            "frac": round(ach / peak_c, 4)}


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML on a background thread."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, index: int, period_s: float = 0.01):
        self.samples = []
        self.period = period_s
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self.t.join()

    def summary(self, t0=None, t1=None):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        win = [s for s in self.samples if (t0 is None or s[0] >= t0) and (t1 is None or s[0] <= t1)]
        where = "timed"
        if len(win) < 3:
            win, where = self.samples, "warmup+timed"
        reasons = set()
        for _, _, rs in win:
            for bit, name in self.REASONS.items():
                if rs & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(m for _, m, _ in win), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(win), "window": where}


# ------------------------------------------------------------------ workloads

class Workload:
    """A workload: seeded host inputs and a function that runs one step."""

    def __init__(self, name: str):
        self.name = name
        if name == "depthwise":
            s = wl.DEPTHWISE
            self.shape = s
            self.host = inputs.conv_inputs(s.N, s.C, s.H, s.W, s.K, s.R, s.S, s.groups,
                                           wl.SEEDS["depthwise"], x_dist="normal", w_bound=1 / 3)
        elif name == "tiny_grouped":
            s = wl.TINY_GROUPED
            self.shape = s
            self.host = inputs.conv_inputs(s.N, s.C, s.H, s.W, s.K, s.R, s.S, s.groups,
                                           wl.SEEDS["tiny_grouped"], x_dist="uniform11",
                                           w_bound=1 / math.sqrt(18))
        elif name == "dense_5x9":
            s = wl.DENSE_5X9
            self.shape = s
            self.host = inputs.conv_inputs(s.N, s.C, s.H, s.W, s.K, s.R, s.S, 1,
                                           wl.SEEDS["dense_5x9"], x_dist="uniform01",
                                           w_bound=1 / math.sqrt(1440))
        elif name == "fused_chain":
            s = wl.FUSED_CHAIN.conv
            self.shape = s
            d = inputs.chain_inputs(s.N, s.C, s.H, s.W, s.K, s.R, s.S, 1, wl.FUSED_CHAIN.gn_groups,
                                    seed=wl.SEEDS["fused_chain"])
            self.host = d
        elif name.startswith("ring"):
            N, C, H, W, K, R, pad, g = wl.THRESHOLD_RING[int(name[4:])]
            s = wl.ConvShape(N=N, C=C, H=H, W=W, K=K, R=R, S=R, stride=1, pad=pad, groups=g)
            self.shape = s
            self.host = inputs.conv_inputs(s.N, s.C, s.H, s.W, s.K, R, R, g, 5000 + int(name[4:]),
                                           x_dist="normal", w_bound=1 / math.sqrt(R * R * s.cpg))
        elif name.startswith("sweep"):
            i = int(name[5:])
            s = wl.sweep80()[i]
            self.shape = s
            self.host = inputs.conv_inputs(s.N, s.C, s.H, s.W, s.K, 3, 3, s.groups, wl.sweep_seed(i),
                                           x_dist="normal", w_bound=1 / math.sqrt(9 * s.cpg))
        else:
            raise ValueError(name)
        self.chain = name == "fused_chain"

    @property
    def bytes(self) -> int:
        return wl.FUSED_CHAIN.bytes if self.chain else self.shape.bytes

    @property
    def flops(self) -> int:
        return self.shape.flops

    @property
    def kernels_per_step(self) -> int:
        return 3 if self.chain else 1

    def config(self):
        s = self.shape
        c = {"workload": self.name, "x": [s.N, s.C, s.H, s.W], "w": [s.K, s.cpg, s.R, s.S],
             "y": [s.N, s.K, s.P, s.Q], "groups": s.groups, "stride": s.stride, "pad": s.pad,
             "dilation": s.dil}
        if self.chain:
            c["gn_groups"] = wl.FUSED_CHAIN.gn_groups
        return c


class DeviceRunner:
    """Device buffers (a rotating pool larger than L2) and the step call."""

    def __init__(self, wk: Workload, device, l2_bytes: int):
        import torch
        import depthwise_convolution_fp32_b200 as gc
        self.gc = gc
        self.wk = wk
        self.torch = torch
        s = wk.shape
        h = wk.host
        self.w = h["w"].to(device)
        self.K, self.P, self.Q = s.K, s.P, s.Q
        per_set = (h["x"].numel() + s.n_out) * 4
        # one set already larger than L2, or enough sets to cover 4 x L2
        self.n_sets = 1 if per_set >= l2_bytes else math.ceil(4 * l2_bytes / per_set)
        # two pooled allocations sliced into per-set views (16-byte aligned slices)
        xn = (h["x"].numel() + 3) // 4 * 4
        yn = (s.n_out + 3) // 4 * 4
        xpool = torch.empty(self.n_sets * xn, device=device)
        ypool = torch.empty(self.n_sets * yn, device=device)
        x0 = h["x"].to(device).reshape(-1)
        xpool.view(self.n_sets, xn)[:, :x0.numel()].copy_(x0.expand(self.n_sets, -1))
        self.xs = [xpool[i * xn:i * xn + x0.numel()].view(h["x"].shape) for i in range(self.n_sets)]
        self.ys = [ypool[i * yn:i * yn + s.n_out].view(s.N, s.K, s.P, s.Q) for i in range(self.n_sets)]
        self.pool_bytes = self.n_sets * per_set
        if wk.chain:
            self.bias = (h["b_conv"] + h["b_extra"]).to(device)
            self.scale = h["scale"].to(device)
            self.gamma = h["gamma"].to(device)
            self.beta = h["beta"].to(device)
        else:
            self.bias = h["bias"].to(device) if "bias" in h else None

    def step(self, i: int, x=None, y=None, w=None):
        s = self.wk.shape
        x = self.xs[i % self.n_sets] if x is None else x
        y = self.ys[i % self.n_sets] if y is None else y
        w = self.w if w is None else w
        if self.wk.chain:
            self.gc.conv2d_bias_scale_sigmoid_groupnorm(
                x, w, self.bias, self.scale, wl.FUSED_CHAIN.gn_groups, self.gamma, self.beta,
                1e-5, s.stride, s.pad, s.dil, s.groups, out=y)
        else:
            self.gc.conv2d(x, w, self.bias, s.stride, s.pad, s.dil, s.groups, out=y)
        return y


class TimedGraph:
    """`n` calls of `body(i)` captured in one CUDA graph and timed by two
    event record nodes inside it, so the graph's own launch and completion
    stay outside the interval.

    With `lead_in` = 1 one untimed call runs first and the first event is
    recorded on a side branch that waits for that call only: the interval then
    runs from the lead-in call's completion to the n-th timed call's, i.e.
    exactly n calls in steady state, each launched behind its predecessor
    (dependent launch) as in a longer sequence.  Without it the first timed
    call pays its whole launch latency after the event, about 6.5 us more per
    replay.  The first replay (graph upload) is untimed."""

    def __init__(self, body, n, stream, lead_in=1):
        import torch
        self.torch = torch
        self.stream = stream
        self.e0 = torch.cuda.Event(enable_timing=True, external=True)
        self.e1 = torch.cuda.Event(enable_timing=True, external=True)
        self.g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(stream):
            with torch.cuda.graph(self.g, stream=stream):
                for i in range(lead_in):
                    body(n + i)
                side.wait_stream(stream)
                self.e0.record(side)
                for i in range(n):
                    body(i)
                stream.wait_stream(side)
                self.e1.record(stream)
        torch.cuda.synchronize()
        self.replay_ms()

    def replay_ms(self) -> float:
        torch = self.torch
        with torch.cuda.stream(self.stream):
            self.g.replay()
        torch.cuda.synchronize()
        return self.e0.elapsed_time(self.e1)


def time_graph(runner: DeviceRunner, steps: int, warmup: int, dist_barrier):
    """Capture exactly `steps` calls in one CUDA graph; time one replay."""
    torch = runner.torch
    for i in range(warmup):
        runner.step(i)
    torch.cuda.synchronize()
    tg = TimedGraph(runner.step, steps, torch.cuda.Stream())
    dist_barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ms = tg.replay_ms()
    t1 = time.perf_counter()
    dist_barrier()
    del tg
    return ms, t0, t1


def time_e2e(runner: DeviceRunner, steps: int, warmup: int, dist_barrier):
    """Per step: pinned host-to-device copy of the step's inputs (x and w), the
    call through the public API, and the device-to-host copy of its output.
    Steps are pipelined over three streams with a ring of device and pinned
    host buffers (4 deep, 2 for steps over 64 MB), so uploads, calls and
    downloads of neighbouring steps overlap (the two copy directions have their own copy engines);
    every step still moves all of its bytes inside the timed region."""
    torch = runner.torch
    h = runner.wk.host
    # pipeline depth: 4 for small steps (71 -> 82 GB/s on the headline), 2 when a
    # step moves more than 64 MB (the pinned host buffers would reach gigabytes)
    step_bytes = (h["x"].numel() + runner.ys[0].numel()) * 4
    nb = int(os.environ.get("GCONV_E2E_BUFFERS", "4" if step_bytes <= 64 * 2**20 else "2"))
    x_host = [h["x"].pin_memory() for _ in range(nb)]
    w_host = [h["w"].pin_memory() for _ in range(nb)]
    y_host = [torch.empty(runner.ys[0].shape, dtype=torch.float32).pin_memory() for _ in range(nb)]
    # one device buffer per ring slot (the rotating pool may hold a single set)
    x_dev = [torch.empty_like(runner.xs[0]) for _ in range(nb)]
    y_dev = [torch.empty_like(runner.ys[0]) for _ in range(nb)]
    w_dev = [torch.empty_like(runner.w) for _ in range(nb)]
    s_in, s_cp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(nb)]
    ev_cp = [torch.cuda.Event() for _ in range(nb)]
    ev_out = [torch.cuda.Event() for _ in range(nb)]

    def one(i, first):
        b = i % nb
        with torch.cuda.stream(s_in):
            if not first:
                s_in.wait_event(ev_cp[b])        # the call nb steps back is done with x_dev[b], w_dev[b]
            x_dev[b].copy_(x_host[b], non_blocking=True)
            w_dev[b].copy_(w_host[b], non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_cp):
            s_cp.wait_event(ev_in[b])
            if not first:
                s_cp.wait_event(ev_out[b])       # the download nb steps back is done with y_dev[b]
            runner.step(i, x=x_dev[b], y=y_dev[b], w=w_dev[b])
            ev_cp[b].record(s_cp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cp[b])
            y_host[b].copy_(y_dev[b], non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(max(warmup, nb)):
        one(i, i < nb)
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    dist_barrier()
    torch.cuda.synchronize()
    ev0.record(s_in)
    for i in range(steps):
        one(i, i < nb)
    ev1.record(s_out)
    torch.cuda.synchronize()
    dist_barrier()
    ms = ev0.elapsed_time(ev1)
    h2d = (x_host[0].numel() + w_host[0].numel()) * 4
    d2h = y_host[0].numel() * 4
    return ms, h2d, d2h


def time_sync_api(runner: DeviceRunner, steps: int):
    torch = runner.torch
    lat = []
    for i in range(steps):
        t0 = time.perf_counter()
        runner.step(i)
        torch.cuda.current_stream().synchronize()
        lat.append(time.perf_counter() - t0)
    return statistics.median(lat) * 1e6


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_oracle_rate(wk: Workload, budget_s: float, threads: int = 0):
    """Time the FP64 oracle, as it stands, on this host's cores (all of them, or
    `threads`) on a bounded sample of the workload; returns (GB/s, sample
    description, threads used)."""
    import oracle
    oracle.set_num_threads(threads if threads > 0 else (os.cpu_count() or 1))
    s = wk.shape
    h = wk.host
    x = h["x"].numpy()
    w = h["w"].numpy()
    # sample: the first n_b batch items (whole images), grown until the budget
    if wk.chain:
        ch = wl.FUSED_CHAIN
        pairs_all = [(n, G) for n in range(s.N) for G in range(ch.gn_groups)]
        done = 0
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < budget_s and done < len(pairs_all):
            nxt = pairs_all[done:done + 8]
            oracle.chain(x, w, h["b_conv"], h["b_extra"], h["scale"], ch.gn_groups, h["gamma"],
                         h["beta"], 1e-5, s.stride, s.pad, s.dil, s.groups, pairs=nxt)
            done += len(nxt)
        dt = time.perf_counter() - t0
        frac = done / len(pairs_all)
        desc = f"{done} of {len(pairs_all)} (n, GroupNorm group) blocks of the full workload"
    else:
        per_item = 1
        t0 = time.perf_counter()
        done = 0
        passes = 0
        while time.perf_counter() - t0 < budget_s:
            n0 = done % s.N
            n1 = min(s.N, n0 + per_item)
            oracle.conv2d(x[n0:n1], w, h.get("bias"), s.stride, s.pad, s.dil, s.groups)
            done += n1 - n0
            passes += 1
            if passes == 1 and time.perf_counter() - t0 < budget_s / 20:
                per_item = min(s.N, per_item * 4)
        dt = time.perf_counter() - t0
        frac = done / s.N
        desc = f"{done} batch items of N={s.N} (whole images, repeated as needed)"
    gbs = wk.bytes * frac / dt / 1e9
    return gbs, desc, oracle.num_threads()


def bootstrap_ci(samples, reps=2000, seed=0):
    """95% bootstrap interval of the mean of `samples`."""
    a = np.asarray(samples, dtype=np.float64)
    rng = np.random.default_rng(seed)
    means = a[rng.integers(0, len(a), (reps, len(a)))].mean(axis=1)
    return float(np.percentile(means, 2.5)), float(np.percentile(means, 97.5))


def torch_conv_graph_us(r, per_batch, batches):
    """PyTorch's own FP32 conv2d (cuDNN, autotuned, TF32 off) on the same
    rotating inputs, timed the same way (a CUDA graph of per_batch calls):
    the comparison the pages make against tuned PyTorch."""
    import torch
    import torch.nn.functional as F
    s = r.wk.shape
    prev = (torch.backends.cudnn.benchmark, torch.backends.cudnn.allow_tf32)
    torch.backends.cudnn.benchmark, torch.backends.cudnn.allow_tf32 = True, False
    try:
        def call(i):
            return F.conv2d(r.xs[i % r.n_sets], r.w, r.bias, s.stride, s.pad, s.dil, s.groups)
        for i in range(3):
            call(i)
        torch.cuda.synchronize()
        tg = TimedGraph(call, per_batch, torch.cuda.Stream())
        us = [tg.replay_ms() * 1e3 / per_batch for b in range(batches)]
        del tg
        return statistics.mean(us)
    finally:
        torch.backends.cudnn.benchmark, torch.backends.cudnn.allow_tf32 = prev


def write_records(args, gc, device, l2, hbm_peak, meas, batches=10, per_batch=30):
    """One record per shape: kernel chosen, status, graph-device and synchronized-API
    latency (mean over 10 batches of 30 calls, 95% bootstrap interval), GB/s,
    GFLOP/s and the binding roofline term."""
    import torch
    names = ["tiny_grouped", "depthwise", "fused_chain", "dense_5x9"] + [f"sweep{i}" for i in range(80)]
    out = []
    for nm in names:
        wk = Workload(nm)
        s = wk.shape
        plan = gc.plan_name(s.N, s.C, s.H, s.W, s.K, s.R, s.S, s.stride, s.pad, s.dil, s.groups, wk.chain)
        rec = {"workload": nm, "shape": s.label(), "kernel": plan, "bytes": wk.bytes, "flops": wk.flops}
        if plan in ("unsupported", "invalid"):
            rec["status"] = plan
            out.append(rec)
            continue
        r = DeviceRunner(wk, device, l2)
        for i in range(3):
            r.step(i)
        torch.cuda.synchronize()
        tg = TimedGraph(r.step, per_batch, torch.cuda.Stream())
        graph_us = [tg.replay_ms() * 1e3 / per_batch for b in range(batches)]
        del tg
        sync_us = []
        for b in range(batches):
            lat = []
            for i in range(per_batch):
                t0 = time.perf_counter()
                r.step(i)
                torch.cuda.current_stream().synchronize()
                lat.append(time.perf_counter() - t0)
            sync_us.append(statistics.mean(lat) * 1e6)
        gm = statistics.mean(graph_us)
        sm = statistics.mean(sync_us)
        rec.update({
            "status": "measured",
            "graph_us": round(gm, 3), "graph_ci95": [round(v, 3) for v in bootstrap_ci(graph_us)],
            "sync_us": round(sm, 3), "sync_ci95": [round(v, 3) for v in bootstrap_ci(sync_us)],
            "GB/s": round(wk.bytes / gm / 1e3, 1), "GFLOP/s": round(wk.flops / gm / 1e3, 1),
            "roofline": roofline_for(wk, gm * 1e-6, plan, hbm_peak, meas),
            "pool_sets": r.n_sets,
        })
        if not wk.chain:
            tg = torch_conv_graph_us(r, per_batch, batches)
            rec.update({"torch_graph_us": round(tg, 3), "speedup_vs_torch": round(tg / gm, 3)})
        out.append(rec)
        del r
        torch.cuda.empty_cache()
    with open(args.records, "w") as f:
        json.dump({"device": torch.cuda.get_device_name(device), "hbm_peak_gbs": hbm_peak,
                   "kernel_family": args.force_kernel, "batches": batches, "per_batch": per_batch,
                   "records": out}, f, indent=1)
    print(json.dumps({"records": len(out), "file": args.records}))




def tuning_workloads():
    out = [Workload(n) for n in ("tiny_grouped", "depthwise", "fused_chain", "dense_5x9")]
    out += [Workload(f"sweep{i}") for i in range(80)]
    for j, (N, C, H, W, K, R, pad, g) in enumerate(wl.THRESHOLD_RING):
        out.append(Workload(f"ring{j}"))
    return out


def candidate_families(gc, s, chain):
    """Kernel families (force names) that can run the shape, direct ones per
    channels-per-thread choice."""
    c = []
    for fam in ("direct_stream", "direct_blocked"):
        if chain and fam == "direct_stream":
            continue
        kpg = s.K // s.groups
        for kt in (1, 2, 4, 8):
            if kpg % kt:
                continue
            if chain and (wl.FUSED_CHAIN.conv.K // wl.FUSED_CHAIN.gn_groups) % kt and \
                    kt % (wl.FUSED_CHAIN.conv.K // wl.FUSED_CHAIN.gn_groups):
                continue
            name = f"{fam}:kt{kt}"
            gc.force_kernel(name)
            plan = gc.plan_name(s.N, s.C, s.H, s.W, s.K, s.R, s.S, s.stride, s.pad, s.dil, s.groups, chain)
            if plan not in ("unsupported", "invalid") and (fam != "direct_stream" or "stream" in plan):
                c.append(name)
    for fam in ("igemm_split", "igemm_fused"):
        gc.force_kernel(fam)
        if gc.plan_name(s.N, s.C, s.H, s.W, s.K, s.R, s.S, s.stride, s.pad, s.dil, s.groups, chain).startswith("igemm"):
            c.append(fam)
    gc.force_kernel("winograd")
    if gc.plan_name(s.N, s.C, s.H, s.W, s.K, s.R, s.S, s.stride, s.pad, s.dil, s.groups, chain).startswith("winograd"):
        c.append("winograd")
    gc.force_kernel("auto")
    return c


def write_dispatch_table(args, gc, device, l2, batches=3, per_batch=20):
    """Per tuning shape: time every candidate family under the benchmark's own
    graph timing (rotating buffers larger than L2, `per_batch` calls per graph,
    mean over `batches` replays) and keep the fastest.  Candidates within 1% of
    the fastest keep the planner's own default order (streaming, blocked,
    implicit GEMM) so the table only overrides where the measurement says so."""
    import torch
    entries = []
    for wk in tuning_workloads():
        s = wk.shape
        cands = candidate_families(gc, s, wk.chain)
        if not cands:
            continue
        r = DeviceRunner(wk, device, l2)
        us = {}
        for name in cands:
            gc.force_kernel(name)
            try:
                for i in range(3):
                    r.step(i)
                torch.cuda.synchronize()
                tg = TimedGraph(r.step, per_batch, torch.cuda.Stream())
                t = [tg.replay_ms() * 1e3 / per_batch for b in range(batches)]
                del tg
                us[name] = round(statistics.mean(t), 3)
            finally:
                gc.force_kernel("auto")
        fastest = min(us.values())
        best = next(n for n in cands if us[n] <= 1.01 * fastest)   # within 1%: the earlier candidate
        entries.append({"workload": wk.name, "shape": [s.N, s.C, s.H, s.W, s.K, s.R, s.S, s.stride, s.pad, s.dil,
                                                       s.groups],
                        "chain": 1 if wk.chain else 0, "best": best, "us": us})
        print(json.dumps({"workload": wk.name, "best": best, "us": us[best]}), flush=True)
        del r
        torch.cuda.empty_cache()
    with open(args.dispatch_table, "w") as f:
        json.dump({"about": "per-shape kernel choice measured on B200 with bench.py --dispatch-table: graph "
                            "device time per call (rotating buffers larger than L2), every family that can "
                            "run the shape; 'best' is compiled into libgconv.so, other shapes follow the "
                            "planner's rules",
                   "device": torch.cuda.get_device_name(device), "batches": batches, "per_batch": per_batch,
                   "entries": entries}, f, indent=1)


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="depthwise")
    ap.add_argument("--no-shapes", action="store_true",
                    help="skip the other page workloads (tiny grouped, depthwise, chain, dense) and the "
                         "80-shape sweep")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--records", default=None,
                    help="write per-shape records (page workloads + 80-shape sweep) to this JSON file "
                         "and exit: 10 batches x 30 calls per boundary, 95%% bootstrap intervals")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-block", action="store_true",
                    help="skip the MobileNetV2 block timing (depthwise workload only)")
    ap.add_argument("--force-kernel", default="auto",
                    help="kernel family for A/B runs: auto, direct, direct_cpasync, generic, igemm")
    ap.add_argument("--profile", action="store_true",
                    help="profiler target: run --calls eager calls of --workload (at --batch), each "
                         "followed by a synchronize, print one line and exit (no timing)")
    ap.add_argument("--batch", type=int, default=0, help="--profile: override N (0: the workload's own)")
    ap.add_argument("--calls", type=int, default=2, help="--profile: number of calls")
    ap.add_argument("--dispatch-table", default=None,
                    help="time every kernel family (and direct-kernel channels per thread) on the tuning "
                         "shapes (page workloads, 80-shape sweep, shapes around the implicit-GEMM "
                         "threshold) and write the per-shape choices to this JSON file "
                         "(depthwise_convolution_fp32_b200/dispatch_table.json is the compiled-in copy)")
    ap.add_argument("--profile-graph", action="store_true",
                    help="profiler target: capture --steps calls of --workload (rotating buffers, as the "
                         "timed region) in one CUDA graph and replay it once inside the NVTX range "
                         "'gconv_graph' (ncu --nvtx --nvtx-include gconv_graph/ --graph-profiling graph)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, rank)

    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)

    def barrier():
        if world > 1:
            dist.barrier()

    from depthwise_convolution_fp32_b200 import build
    build.build()
    import depthwise_convolution_fp32_b200 as gc
    gc.library()
    gc.force_kernel(args.force_kernel)

    props = torch.cuda.get_device_properties(device)
    l2 = getattr(props, "L2_cache_size", 126 * 2 ** 20) or 126 * 2 ** 20
    hbm_peak, peak_kind, meas = peaks()
    if not (args.profile or args.profile_graph):
        measure_compute_peaks()

    if args.records:
        return write_records(args, gc, device, l2, hbm_peak, meas)
    if args.dispatch_table:
        return write_dispatch_table(args, gc, device, l2)
    if args.profile:
        return run_profile_case(args, gc, device)
    if args.profile_graph:
        return run_profile_graph(args, gc, device, l2)

    wk = Workload(args.workload)
    runner = DeviceRunner(wk, device, l2)
    sampler = ClockSampler(local_rank)
    with sampler:
        ms, t0, t1 = time_graph(runner, args.steps, args.warmup, barrier)
        e2e_ms, h2d, d2h = time_e2e(runner, args.steps, args.warmup, barrier)
        sync_us = time_sync_api(runner, min(args.steps, 200))
    clocks = sampler.summary(t0, t1)
    # the same calls on one buffer set that stays in L2 (labelled L2-warm,
    # reported beside the L2-cold headline; only when one set fits in L2)
    warm_ms = None
    if (wk.host["x"].numel() + wk.shape.n_out) * 4 * 2 <= l2:
        warm = DeviceRunner(wk, device, 0)
        warm_ms, _, _ = time_graph(warm, args.steps, args.warmup, barrier)
        del warm

    ms, e2e_ms = max_over_ranks([ms, e2e_ms], device, world)
    per_step_s = ms / 1e3 / args.steps
    value = weak_scaling_rate(wk.bytes, world, args.steps, ms) / 1e9
    e2e_value = weak_scaling_rate(wk.bytes, world, args.steps, e2e_ms) / 1e9
    gflops = weak_scaling_rate(wk.flops, world, args.steps, ms) / 1e9

    # dominant kernel: the convolution (the only kernel of a direct plain conv)
    shp = wk.shape
    plan = gc.plan_name(shp.N, shp.C, shp.H, shp.W, shp.K, shp.R, shp.S, shp.stride, shp.pad, shp.dil,
                        shp.groups, wk.chain)
    roof = roofline_for(wk, per_step_s, plan, hbm_peak, meas)
    roof.update({"traffic": stored_traffic(wk.name), "peak_kind": peak_kind, "kernel": plan})
    launches = wk.kernels_per_step + (2 if plan.startswith("igemm") else 0)

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded)",
        "config": dict(wk.config(), **{
            "l2": f"rotating pool of {runner.n_sets} buffer sets, {runner.pool_bytes / 2**20:.0f} MiB "
                  f"(L2 {l2 / 2**20:.0f} MiB)",
            "timing": "CUDA graph: one untimed lead-in call, then exactly K calls timed by event record nodes in the graph (lead-in completion to K-th completion)",
            "parallelism": f"replicas x{world} (batch shards, no collective)",
            "kernel_family": args.force_kernel}),
        "gflops": round(gflops, 2),
        "sync_api_us": round(sync_us, 2),
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "roofline": roof,
        "l2_warm": None if warm_ms is None else {
            "us_per_step": round(warm_ms * 1e3 / args.steps, 3),
            "GB/s": round(wk.bytes * args.steps / (warm_ms / 1e3) / 1e9, 1),
            "note": "one buffer set reused every call (inputs and outputs resident in L2); the headline "
                    "value is L2-cold"},
        "gpu_launches": launches * args.steps,
        "compute_peaks": dict(MEASURED_COMPUTE, note="microbenchmarks on this GPU, reported beside the "
                              "roofline denominators (alu: unit counts x clock; tensor: bf16 GEMM peak x "
                              "nominal tf32 ratio)", alu_peak_tflops=round(fp32_peak_tflops(), 2),
                              tensor_peak_tflops=round(tensor_fp32_peak_tflops(meas), 2)),
        "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
        "clock_samples": {"n": clocks.get("samples"), "window": clocks.get("window")},
    }

    if not args.no_shapes:
        # every page workload with the headline's fields: graph time, roofline,
        # end-to-end through the public API, synchronous API, CPU oracle baseline
        cfgs = {}
        for nm in ("tiny_grouped", "depthwise", "fused_chain", "dense_5x9"):
            if nm == args.workload:
                continue
            cfgs[nm] = measure_config(nm, gc, device, l2, hbm_peak, meas, barrier, args, rank, world)
            torch.cuda.empty_cache()
        result["configs"] = cfgs
        result["sweep80"] = measure_sweep(gc, device, l2, hbm_peak, meas, barrier)

    if args.workload == "depthwise" and not args.no_block:
        result["mobilenetv2_block"] = measure_block(device, max(20, min(args.steps, 200)), args.warmup)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, desc, thr = cpu_oracle_rate(wk, args.cpu_budget)
        gbs1, _, _ = cpu_oracle_rate(wk, args.cpu_budget / 4, threads=1)
        result["cpu_baseline"] = {"value": round(gbs, 4), "unit": UNIT, "cores": thr,
                                  "kind": "oracle", "sample": desc, "single_thread_value": round(gbs1, 4),
                                  "cpu_model": cpu_model()}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


def measure_config(name, gc, device, l2, hbm_peak, meas, barrier, args, rank, world):
    """One page workload with the headline's fields (fewer calls): device time
    in a CUDA graph, roofline, end-to-end GB/s through the public API with the
    step's host copies, synchronous-API latency and the CPU oracle baseline
    (all host cores and one)."""
    import torch
    wk = Workload(name)
    r = DeviceRunner(wk, device, l2)
    s = wk.shape
    k = max(3, min(args.steps, 20))
    ms, _, _ = time_graph(r, k, 3, barrier)
    sec = ms / 1e3 / k
    plan = gc.plan_name(s.N, s.C, s.H, s.W, s.K, s.R, s.S, s.stride, s.pad, s.dil, s.groups, wk.chain)
    e2e_ms, h2d, d2h = time_e2e(r, k, 3, barrier)
    out = {"label": s.label(), "kernel": plan, "us": round(sec * 1e6, 3),
           "GB/s": round(wk.bytes / sec / 1e9, 1), "GFLOP/s": round(wk.flops / sec / 1e9, 1),
           "roofline": roofline_for(wk, sec, plan, hbm_peak, meas),
           "e2e": {"value": round(wk.bytes * k / (e2e_ms / 1e3) / 1e9, 2), "unit": UNIT,
                   "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
           "sync_api_us": round(time_sync_api(r, k), 2)}
    del r
    # DRAM bytes per call from the committed ncu capture of this workload (all
    # of the call's launches), when it matches the current kernel sources
    out["roofline"]["traffic"] = stored_traffic(name)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, desc, thr = cpu_oracle_rate(wk, max(1.0, args.cpu_budget / 4))
        gbs1, _, _ = cpu_oracle_rate(wk, max(0.5, args.cpu_budget / 8), threads=1)
        out["cpu_baseline"] = {"value": round(gbs, 4), "unit": UNIT, "cores": thr, "kind": "oracle",
                               "sample": desc, "single_thread_value": round(gbs1, 4)}
    return out


def measure_sweep(gc, device, l2, hbm_peak, meas, barrier, k=20):
    """The 80-shape sweep under graph timing (k calls per shape, rotating
    buffers): per-shape time and roofline fraction, and their summary."""
    import torch
    per = []
    for i in range(80):
        wk = Workload(f"sweep{i}")
        s = wk.shape
        r = DeviceRunner(wk, device, l2)
        ms, _, _ = time_graph(r, k, 3, barrier)
        sec = ms / 1e3 / k
        plan = gc.plan_name(s.N, s.C, s.H, s.W, s.K, s.R, s.S, s.stride, s.pad, s.dil, s.groups, False)
        roof = roofline_for(wk, sec, plan, hbm_peak, meas)
        per.append({"i": i, "us": round(sec * 1e6, 3), "MB": round(wk.bytes / 1e6, 2), "kernel": plan,
                    "bound": roof["bound"], "frac": roof["frac"]})
        del r
        torch.cuda.empty_cache()

    def gmean(v):
        v = [x for x in v if x > 0]   # a shape timed at zero (e.g. under a profiler) carries no ratio
        return round(math.exp(sum(math.log(x) for x in v) / len(v)), 4) if v else None
    big = [p["frac"] for p in per if p["MB"] >= 50]
    big_hbm = [p["frac"] for p in per if p["MB"] >= 50 and p["bound"] == "hbm"]
    return {"calls_per_shape": k, "geomean_frac": gmean([p["frac"] for p in per]),
            "geomean_frac_ge_50MB": gmean(big), "geomean_frac_ge_50MB_hbm_bound": gmean(big_hbm),
            "n_ge_50MB": len(big), "n_ge_50MB_at_0.70": sum(1 for f in big if f >= 0.70),
            "shapes": per}


def run_profile_case(args, gc, device):
    """A small, self-contained target for one ncu capture: `--calls` eager calls
    of one workload on the same buffers (optionally at a reduced batch), each
    followed by a synchronize.  Only the library's kernels run after the
    one-time input upload."""
    import dataclasses
    import torch
    wk = Workload(args.workload)
    s = wk.shape
    if args.batch > 0 and args.batch != s.N:
        s = dataclasses.replace(s, N=args.batch)
        wk.shape = s
        wk.host = {k: (v[:args.batch] if k == "x" else v) for k, v in wk.host.items()}
        if wk.host["x"].shape[0] < args.batch:
            raise SystemExit(f"--batch {args.batch} exceeds the workload's N")
    r = DeviceRunner(wk, device, 0)
    y = None
    for i in range(args.calls):
        y = r.step(0)
        torch.cuda.synchronize()
    plan = gc.plan_name(s.N, s.C, s.H, s.W, s.K, s.R, s.S, s.stride, s.pad, s.dil, s.groups, wk.chain)
    print(f"{args.workload} {s.label()} plan={plan} calls={args.calls} "
          f"mean|y|={float(y.abs().mean()):.6f}", flush=True)


def run_profile_graph(args, gc, device, l2):
    """The timed region of the benchmark as one profiler workload: --steps calls
    over the rotating buffer pool captured in one CUDA graph, uploaded by one
    untimed replay, then replayed once inside the NVTX range 'gconv_graph'.
    Only that replay falls inside the range."""
    import torch
    wk = Workload(args.workload)
    r = DeviceRunner(wk, device, l2)
    r.step(0)                      # one eager call: workspace and plans ready before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        with torch.cuda.graph(g, stream=st):
            for i in range(args.steps):
                r.step(i)
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("gconv_graph")
    with torch.cuda.stream(st):
        g.replay()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    del g
    print(f"{args.workload} graph of {args.steps} calls over {r.n_sets} buffer sets "
          f"({r.pool_bytes / 2**20:.0f} MiB)", flush=True)


def measure_block(device, steps, warmup):
    """One MobileNetV2 inverted-residual block x[4,24,56,56] (1x1 24->144, BN,
    ReLU6, depthwise 3x3, BN, ReLU6, 1x1 144->24, residual add), forward with
    PyTorch's depthwise convolution, with this library's, and with this
    library's depthwise convolution + BatchNorm + ReLU6 in one call, timed both ways
    the pages distinguish: `steps` forwards replayed from one CUDA graph
    (device events), and eager forwards each followed by a synchronize
    (host clock).  Activations stay L2-resident for both variants alike."""
    import torch
    from depthwise_convolution_fp32_b200 import block
    prm = inputs.mobilenet_block_inputs(wl.SEEDS["depthwise"] + 1)
    x = prm.pop("x").to(device)
    prm = block.to_device(prm, device)
    out = {}
    folded = block.fold_bn(prm["bn2"])
    variants = (("library", lambda: block.forward(x, prm, block.library_depthwise)),
                ("library_fused_bn_relu6", lambda: block.forward_fused(x, prm, folded)),
                ("torch", lambda: block.forward(x, prm, block.torch_depthwise)))
    for name, fwd in variants:
        for _ in range(max(3, warmup)):
            fwd()
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            fwd()
        torch.cuda.synchronize()
        tg = TimedGraph(lambda i: fwd(), steps, s)
        graph_us = tg.replay_ms() * 1e3 / steps
        del tg
        n_sync = max(20, steps // 2)
        t0 = time.perf_counter()
        for _ in range(n_sync):
            fwd()
            torch.cuda.synchronize()
        sync_us = (time.perf_counter() - t0) * 1e6 / n_sync
        out[name] = (graph_us, sync_us)
    y_lib = block.forward(x, prm, block.library_depthwise)
    y_fused = block.forward_fused(x, prm, folded)
    y_ref = block.forward(x, prm, block.torch_depthwise)
    return {"x": list(x.shape), "graph_us": {k: round(v[0], 3) for k, v in out.items()},
            "sync_us": {k: round(v[1], 3) for k, v in out.items()},
            "speedup_graph": round(out["torch"][0] / out["library"][0], 3),
            "speedup_sync": round(out["torch"][1] / out["library"][1], 3),
            "speedup_graph_fused": round(out["torch"][0] / out["library_fused_bn_relu6"][0], 3),
            "speedup_sync_fused": round(out["torch"][1] / out["library_fused_bn_relu6"][1], 3),
            "max_abs_diff_vs_torch": float((y_lib - y_ref).abs().max()),
            "max_abs_diff_fused_vs_torch": float((y_fused - y_ref).abs().max()),
            "pages_reported": {"speedup_graph": 1.14, "speedup_sync": 0.68, "gpu": "RTX 4090"}}


def run_reference(args, rank):
    """The reference arm: the FP64 CPU oracle, as it stands, on this host."""
    if rank != 0:
        return
    wk = Workload(args.workload)
    budget = max(2.0, min(20.0, args.cpu_budget))
    rates = []
    for _ in range(args.warmup):
        cpu_oracle_rate(wk, budget / 10)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        r, desc, thr = cpu_oracle_rate(wk, budget / max(1, args.steps))
        rates.append(r)
    wall = time.perf_counter() - t0
    value = statistics.median(rates)
    ms_per_step = wall * 1e3 / args.steps
    result = {
        "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "impl": "reference", "config": wk.config(),
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": thr, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(result), flush=True)


if __name__ == "__main__":
    main()
