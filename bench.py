#!/usr/bin/env python
"""Benchmark of the DeformConv1d forward on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME|all] [--impl ours|reference]

A step is one full forward pass (sampling, interpolation, mask, contraction, bias, store)
over one batch of the named synthetic workload (default: the large dense strided bf16
workload, B=32, C=1024, K=9, stride 2, dilation 2, groups 4, L=8192, the largest of the
five).  Inputs are resident in HBM before the timed
region; L2 is flushed (a 256 MiB write) between steps, outside the timed events; each step
is timed with CUDA events on the launching stream, with a barrier and a device
synchronisation on both sides of the K timed steps, and the time is the max over ranks.
Under torchrun each rank runs its own batch (weak scaling, no collective on the data path).

``--impl reference`` times the CPU oracle instead (rank 0 only), on bounded samples of the
same workload.  ``--pass backward`` prints one line for the backward pass instead (all
gradients of one batch per step; the work counted is its two contractions).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "DeformConv1d forward TFLOP/s (HBM GB/s if depthwise) as % of B200 roofline"
METRIC_BACKWARD = "DeformConv1d backward TFLOP/s as % of B200 roofline"
METRIC_PACKED = "PackedDeformConv1d forward TFLOP/s (trunk + deformable conv)"
DEFAULT_WORKLOAD = "large_bf16"
L2_FLUSH_BYTES = 256 << 20

# Fallback denominators (used only when MEASURED_PEAKS.json is absent).
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# fp32 FFMA ALU peak: 148 SMs x 128 fp32 lanes x 2 flop x 1965 MHz (clocks.max.sm).
ALU_F32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
# Nominal dense tensor ratios to bf16 (2.25 PFLOP/s): tf32 1.1 PFLOP/s.
TF32_OVER_BF16 = 1.1 / 2.25


# ------------------------------------------------------------------ peaks and roofline

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def roofline_for(kernel: str, w: W.Workload, peaks: dict):
    """(bound, unit, peak, algorithmic amount per launch, note) of the step's main kernel."""
    flops = w.flops() / 1e12
    gbytes = w.algorithmic_bytes() / 1e9
    src = peaks["source"]
    if kernel.startswith("depthwise"):
        return "hbm", "GB/s", peaks["hbm_gbs"], gbytes, f"HBM copy bandwidth ({src})"
    if kernel.startswith("tcgen05_bf16"):
        return "tensor", "TFLOP/s", peaks["bf16_tflops"], flops, f"bf16 dense GEMM burst ({src})"
    if kernel.startswith("tcgen05_f16"):
        return ("tensor", "TFLOP/s", peaks["bf16_tflops"], flops,
                f"bf16 dense GEMM burst ({src}) x 1 (fp16 and bf16 share the nominal dense rate)")
    if kernel.startswith("tcgen05_3xtf32"):
        # The fp32-exact contraction against the TF32 dense peak with its flops counted
        # once (each product costs three TF32 passes; that ceiling is reported apart).
        pk = peaks["bf16_tflops"] * TF32_OVER_BF16
        return ("tensor", "TFLOP/s", pk, flops,
                f"tf32 dense peak (bf16 burst {src} x 1.1/2.25 nominal), flops counted once")
    return "alu", "TFLOP/s", ALU_F32_TFLOPS, flops, "fp32 FFMA: 148 SMs x 128 lanes x 2 x 1965 MHz"


def pipelined_e2e(dev, pinned: dict, out_shape, out_dtype, launch, steps: int, warmup: int,
                  ws: int):
    """End-to-end time per step through the public API: every step copies its inputs in from
    pinned host memory, runs `launch(inputs, out, stream)` and copies its output back.  Steps
    are pipelined as a user streaming batches would run them: copies in on one stream, the
    forward on another, copies out on a third (the two copy directions use separate copy
    engines), with two device buffer sets, so step i+1's inputs travel while step i computes
    and its output travels back.  Returns ms per step (max over ranks); the whole K-step
    pipeline is timed between one event before it and one after its last copy out."""
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    bufs = [{k: (torch.empty(v.shape, dtype=v.dtype, device=dev) if v is not None else None)
             for k, v in pinned.items()} for _ in range(2)]
    outs = [torch.empty(out_shape, dtype=out_dtype, device=dev) for _ in range(2)]
    hosts = [torch.empty(out_shape, dtype=out_dtype).pin_memory() for _ in range(2)]

    def run(n):
        done_comp, done_out = [], []
        for i in range(n):
            j = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(done_comp[i - 2])   # buffer j's inputs are free
                for k, v in pinned.items():
                    if v is not None:
                        bufs[j][k].copy_(v, non_blocking=True)
                e_in = torch.cuda.Event()
                e_in.record(s_in)
            s_comp.wait_event(e_in)
            if i >= 2:
                s_comp.wait_event(done_out[i - 2])      # buffer j's output was copied out
            launch(bufs[j], outs[j], s_comp)
            e_c = torch.cuda.Event()
            e_c.record(s_comp)
            done_comp.append(e_c)
            with torch.cuda.stream(s_out):
                s_out.wait_event(e_c)
                hosts[j].copy_(outs[j], non_blocking=True)
                e_o = torch.cuda.Event()
                e_o.record(s_out)
            done_out.append(e_o)
        return done_out

    run(max(warmup, 1))
    torch.cuda.synchronize(dev)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize(dev)
    start.record(s_in)
    s_comp.wait_event(start)
    s_out.wait_event(start)
    last = run(steps)[-1]
    s_out.wait_event(last)
    end.record(s_out)
    torch.cuda.synchronize(dev)
    barrier(ws)
    return max_over_ranks(start.elapsed_time(end), ws) / steps


def load_traffic(kernel: str, w: W.Workload):
    """DRAM bytes per launch from the committed ncu summary, if taken on this kernel source."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    for line in lines:
        if not line.strip() or line.startswith("#"):
            continue
        parts = line.split()
        if len(parts) < 4 or parts[0] != kernel or parts[1] != w.name:
            continue
        src = os.path.join(ROOT, "deformable_convolution_dcn1d_b200", "csrc", parts[3])
        want = parts[4] if len(parts) > 4 else None
        try:
            h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        except OSError:
            return None
        if want is not None and h != want:
            return None   # the kernel changed since the counters were taken
        full = W.WORKLOADS.get(w.name)
        # the recorded figure is per launch of the named workload; a batch override scales it
        return float(parts[2]) * (w.B / full.B if full is not None else 1.0)
    return None


# ------------------------------------------------------------------ clocks during the region

class ClockSampler:
    """Polls NVML (SM clock, throttle reasons) every few ms while the timed region runs."""

    REASONS = [("gpu_idle", "nvmlClocksEventReasonGpuIdle"),
               ("applications_clocks_setting", "nvmlClocksEventReasonApplicationsClocksSetting"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("sync_boost", "nvmlClocksEventReasonSyncBoost"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown")]

    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, attr in self.REASONS:
                    if bits & getattr(nv, attr, 0):
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        # Re-entrant: each timed region of a run adds its samples to the same record.
        if self.nv is not None:
            self._stop.clear()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ distributed plumbing

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, ws: int, device: str = "cuda") -> float:
    if ws == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(ws: int):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ the CPU oracle baseline

def time_oracle(w: W.Workload, inputs: dict, target_s: float, seed: int = 0):
    """Time the oracle on a bounded random sample of the workload's outputs."""
    import numpy as np
    import oracle
    per_point_flops = 2 * (w.C_in // w.groups) * w.K
    total_points = w.B * w.C_out * w.L_out
    rng = np.random.default_rng(seed)

    def pts(n):
        return np.stack([rng.integers(0, w.B, n), rng.integers(0, w.C_out, n),
                         rng.integers(0, w.L_out, n)], axis=1)

    args = (inputs["x"], inputs["offsets"], inputs["mask"], inputs["weight"], inputs["bias"],
            w.stride, w.padding, w.dilation, w.groups, w.offset_groups, w.unconstrained)
    n = 256
    while True:
        p = pts(n)
        t0 = time.perf_counter()
        oracle.forward_points(*args, p)
        dt = time.perf_counter() - t0
        if dt > 0.2 or n >= total_points:
            break
        n = min(n * 4, total_points)
    n = int(min(total_points, max(n, n * target_s / max(dt, 1e-9))))
    p = pts(n)
    t0 = time.perf_counter()
    r = oracle.forward_points(*args, p)
    dt = time.perf_counter() - t0
    return n * per_point_flops / dt / 1e12, n, dt, oracle.threads(), (p, r)


def unit_value(w: W.Workload, kernel: str, seconds: float, ranks: int = 1):
    """Whole-job throughput in the metric's unit."""
    if kernel.startswith("depthwise"):
        return ranks * w.algorithmic_bytes() / seconds / 1e9, "GB/s"
    return ranks * w.flops() / seconds / 1e12, "TFLOP/s"


# ------------------------------------------------------------------ the two arms

def run_reference(args, w: W.Workload):
    ws, rank, _ = dist_env()
    if rank != 0:
        return None
    import oracle
    inputs = W.make_inputs(w, seed=0)
    per_point_flops = 2 * (w.C_in // w.groups) * w.K
    # Calibrate one step to about 1 s of oracle work.
    _, n_step, _, cores, _ = time_oracle(w, inputs, target_s=1.0)
    import numpy as np
    rng = np.random.default_rng(1)
    a = (inputs["x"], inputs["offsets"], inputs["mask"], inputs["weight"], inputs["bias"],
         w.stride, w.padding, w.dilation, w.groups, w.offset_groups, w.unconstrained)

    def step():
        p = np.stack([rng.integers(0, w.B, n_step), rng.integers(0, w.C_out, n_step),
                      rng.integers(0, w.L_out, n_step)], axis=1)
        oracle.forward_points(*a, p)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    depthwise = w.groups == w.C_in == w.C_out
    if depthwise:
        frac = n_step * args.steps / (w.B * w.C_out * w.L_out)
        value, unit = frac * w.algorithmic_bytes() / dt / 1e9, "GB/s"
    else:
        value, unit = n_step * args.steps * per_point_flops / dt / 1e12, "TFLOP/s"
    sample = f"{n_step} random outputs per step of {w.B * w.C_out * w.L_out}"
    return {"metric": METRIC, "value": value, "unit": unit, "impl": "reference",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, "oracle", ws, l2="n/a (CPU)"),
            "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def workload_config(w: W.Workload, kernel: str, ws: int, l2: str):
    return {"workload": w.name, "B": w.B, "C_in": w.C_in, "C_out": w.C_out, "K": w.K,
            "stride": w.stride, "padding": w.padding, "dilation": w.dilation,
            "groups": w.groups, "offset_groups": w.offset_groups, "L_in": w.L_in,
            "L_out": w.L_out, "dtype": w.dtype, "mask": w.mask,
            "unconstrained": w.unconstrained, "kernel": kernel, "l2": l2,
            "parallelism": f"dp{ws} (independent batch per GPU)"}


def run_ours(args, w: W.Workload, peaks: dict, want_cpu: bool):
    import deformable_convolution_dcn1d_b200 as dcn
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dcn.load()

    host = W.make_inputs(w, seed=rank)
    keys = ["x", "offsets", "mask", "weight", "bias"]
    dev_in = {k: (host[k].to(dev) if host[k] is not None else None) for k in keys}
    out = torch.empty((w.B, w.C_out, w.L_out), dtype=w.torch_dtype, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def step(d, o):
        dcn.dcn1d_forward(d["x"], d["offsets"], d["mask"], d["weight"], d["bias"], w.stride,
                          w.padding, w.dilation, w.groups, w.offset_groups, w.unconstrained,
                          out=o, stream=stream)

    kernel = dcn.dcn1d_forward_kernel_name(dev_in["x"], dev_in["offsets"], dev_in["mask"],
                                           dev_in["weight"], dev_in["bias"], w.stride,
                                           w.padding, w.dilation, w.groups, w.offset_groups,
                                           w.unconstrained, out)
    for _ in range(max(args.warmup, 0)):
        flush.zero_()
        step(dev_in, out)
    torch.cuda.synchronize(dev)
    launches_per_step = dcn.dcn1d_last_launch_count()

    # ---- device-resident timing: K steps, events around each whole step
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(ws)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            step(dev_in, out)
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
    barrier(ws)
    ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    ms = max_over_ranks(ms, ws)
    ms_step = ms / args.steps

    # ---- the main kernel's own time: a second run of the same K steps in which the
    # library records events right around its main kernel (the events add a few us to
    # each step, so they stay out of the run that gives the step time above)
    k_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    k_ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for e in k_starts + k_ends:
        e.record(stream)   # creates the CUDA event (torch creates events lazily)
    barrier(ws)
    torch.cuda.synchronize(dev)
    with clk:
        for i in range(args.steps):
            flush.zero_()
            dcn.dcn1d_set_timing_events(k_starts[i], k_ends[i])
            step(dev_in, out)
        torch.cuda.synchronize(dev)
    barrier(ws)
    ms_kernel = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(k_starts, k_ends)),
                               ws) / args.steps
    value, unit = unit_value(w, kernel, ms_step / 1e3, ws)

    # ---- end to end through the public API from pinned host buffers
    pinned = {k: (host[k].pin_memory() if host[k] is not None else None) for k in keys}
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in pinned.values() if v is not None)
    d2h = out_host.numel() * out_host.element_size()

    def launch(d, o, s):
        dcn.dcn1d_forward(d["x"], d["offsets"], d["mask"], d["weight"], d["bias"], w.stride,
                          w.padding, w.dilation, w.groups, w.offset_groups, w.unconstrained,
                          out=o, stream=s)

    # no separate L2 flush between the pipelined steps: each step's inputs arrive by copy
    # from the host through L2 (551 MB a step on the large workload, several times L2)
    with clk:
        e_ms_step = pipelined_e2e(dev, pinned, out.shape, out.dtype, launch, args.steps,
                                  args.warmup, ws)
    e_ms = e_ms_step * args.steps
    e_value, e_unit = unit_value(w, kernel, e_ms / args.steps / 1e3, ws)

    # ---- roofline of the step's kernel (one kernel per step: its time is the step time)
    bound, r_unit, peak, per_launch, note = roofline_for(kernel, w, peaks)
    achieved = per_launch / (ms_kernel / 1e3)
    roof = {"bound": bound, "achieved": achieved, "peak": peak, "unit": r_unit,
            "frac": achieved / peak, "traffic": load_traffic(kernel, w), "kernel": kernel,
            "peak_source": note, "launches_per_step": launches_per_step,
            "kernel_ms": ms_kernel,
            "timing": "CUDA events the library records around its main kernel, per step, "
                      "in a second timed run of the same K steps"}
    if kernel.startswith("tcgen05_3xtf32"):
        # the same time against the ceiling of three TF32 passes per product
        roof["frac_of_3pass_ceiling"] = achieved / (peak / 3.0)

    line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic (seeded, shapes and distributions of the named workload)",
            "config": workload_config(w, kernel, ws,
                                      l2="flushed between steps (256 MiB write outside the timed events)"),
            "roofline": roof,
            "clocks": dict(clk.summary(), region="the three timed runs (step, kernel, e2e)"),
            "e2e": {"value": e_value, "unit": e_unit, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "note": "pinned host inputs copied in, forward, output copied out, every step; "
                            "steps pipelined over two device buffer sets (copies in, forward "
                            "and copies out on three streams)"},
            "gpu_launches": launches_per_step * args.steps}
    if want_cpu and ws == 1 and rank == 0:
        v, n, dt, cores, (pts, r) = time_oracle(w, host, target_s=args.cpu_seconds)
        if kernel.startswith("depthwise"):
            v = n / (w.B * w.C_out * w.L_out) * w.algorithmic_bytes() / dt / 1e9
        # the same sampled outputs of the timed path (out holds the last step's result, on
        # the same inputs): max|y - r| / max|r| over the sample
        y = out.double().cpu().numpy()[pts[:, 0], pts[:, 1], pts[:, 2]]
        den = float(abs(r).max()) if len(r) else 0.0
        err = float(abs(y - r).max()) / den if den > 0 else float(abs(y).max())
        line["cpu_baseline"] = {"value": v, "unit": unit, "cores": cores, "kind": "oracle",
                                "sample": f"{n} random outputs of {w.B * w.C_out * w.L_out} "
                                          f"({dt:.1f} s)",
                                "max_rel_err_of_timed_path": err}
    return line if rank == 0 else None


# ------------------------------------------------------------------ the backward pass

def time_oracle_backward(w: W.Workload, host: dict, gout: torch.Tensor):
    """The oracle's backward on a batch-1 slice of the workload: TFLOP/s, seconds, threads."""
    import oracle
    w1 = w.with_batch(1)
    sl = {k: (v[:1] if (v is not None and k in ("x", "offsets", "mask")) else v)
          for k, v in host.items()}
    t0 = time.perf_counter()
    oracle.backward(sl["x"], sl["offsets"], sl["mask"], sl["weight"], gout[:1], w.stride,
                    w.padding, w.dilation, w.groups, w.offset_groups, w.unconstrained)
    dt = time.perf_counter() - t0
    return 2 * w1.flops() / dt / 1e12, dt, oracle.threads()


def run_backward_pass(args, w: W.Workload, peaks: dict, want_cpu: bool):
    """One backward step = all five gradients of one batch; the work counted is the two
    contractions (2x the forward's flops); the rest (sampling gradient) is overhead."""
    import deformable_convolution_dcn1d_b200 as dcn
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dcn.load()
    host = W.make_inputs(w, seed=rank)
    gout_h = torch.randn(w.B, w.C_out, w.L_out,
                         generator=torch.Generator().manual_seed(100 + rank)).to(host["x"].dtype)
    d = {k: (v.to(dev) if v is not None else None) for k, v in host.items()}
    gout = gout_h.to(dev)
    wanted = tuple(n for n in dcn.GRADS if n != "mask" or d["mask"] is not None)
    like = {"x": d["x"], "offsets": d["offsets"], "mask": d["mask"], "weight": d["weight"]}
    grads = {n: torch.empty((w.C_out,) if n == "bias" else like[n].shape, dtype=d["x"].dtype,
                            device=dev) for n in wanted}
    args_c = (w.stride, w.padding, w.dilation, w.groups, w.offset_groups, w.unconstrained)
    need = dcn.dcn1d_backward_workspace_size(d["x"], d["offsets"], d["mask"], d["weight"], gout,
                                             *args_c, wanted=wanted)
    gemm_kernel = dcn.dcn1d_backward_kernel_name(d["x"], d["offsets"], d["mask"], d["weight"],
                                                 gout, *args_c, wanted=wanted)
    scratch = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def step():
        dcn.dcn1d_backward(d["x"], d["offsets"], d["mask"], d["weight"], gout, *args_c,
                           wanted=wanted, grads=grads, workspace=scratch, stream=stream)

    for _ in range(max(args.warmup, 0)):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    launches = dcn.dcn1d_last_launch_count()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(ws)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
    barrier(ws)
    ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), ws) / args.steps
    per_gpu = 2 * w.flops() / (ms / 1e3) / 1e12
    if gemm_kernel == "tcgen05_gemm" and w.dtype == "f32":   # three TF32 products
        pk = peaks["bf16_tflops"] * TF32_OVER_BF16
        roof = {"bound": "tensor", "achieved": per_gpu, "peak": pk,
                "unit": "TFLOP/s", "frac": per_gpu / pk, "traffic": None,
                "kernel": "backward: two tcgen05 3xTF32 GEMMs (fp32-accurate) + sampling "
                          "gradient + transposes",
                "peak_source": f"tf32 dense peak (bf16 burst {peaks['source']} x 1.1/2.25 "
                               f"nominal), flops counted once",
                "frac_of_3pass_ceiling": per_gpu / (pk / 3.0)}
    elif gemm_kernel == "tcgen05_gemm":   # 16-bit operands on the tensor cores
        roof = {"bound": "tensor", "achieved": per_gpu, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": per_gpu / peaks["bf16_tflops"], "traffic": None,
                "kernel": "backward: two tcgen05 GEMMs (16-bit operands, fp32 accumulation) "
                          "+ sampling gradient + transposes",
                "peak_source": f"bf16 dense GEMM burst ({peaks['source']})"}
    else:
        roof = {"bound": "alu", "achieved": per_gpu, "peak": ALU_F32_TFLOPS,
                "unit": "TFLOP/s", "frac": per_gpu / ALU_F32_TFLOPS, "traffic": None,
                "kernel": "backward: two CUDA-core fp32 GEMMs + sampling gradient",
                "peak_source": "fp32 FFMA: 148 SMs x 128 lanes x 2 x 1965 MHz"}
    roof.update({"launches_per_step": launches,
                 "timing": "CUDA events around the whole backward call, per step"})
    line = {"metric": METRIC_BACKWARD, "value": per_gpu * ws, "unit": "TFLOP/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic (seeded, shapes and distributions of the named workload)",
            "config": workload_config(w, f"backward ({gemm_kernel})", ws,
                                      l2="flushed between steps (256 MiB write outside the timed events)"),
            "roofline": roof,
            "clocks": clk.summary(), "gpu_launches": launches * args.steps,
            "workspace_bytes": need}
    if want_cpu and ws == 1 and rank == 0:
        v, dt, cores = time_oracle_backward(w, host, gout_h)
        line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                "sample": f"all gradients of batch element 0 ({dt:.1f} s)"}
    return line if rank == 0 else None


# ------------------------------------------------------------------ PackedDeformConv1d

PACKED_KEYS = ("x", "dw_weight", "dw_bias", "off_weight", "off_bias", "mask_weight", "mask_bias",
               "weight", "bias")


def packed_flops(w: W.Workload, L_out: int = None, B: int = None) -> int:
    """Multiply-adds x 2 of the layer: the trunk's depthwise (K per channel and position) and
    pointwise heads (C_in per head channel and position), then the deformable convolution."""
    L = w.L_out if L_out is None else L_out
    b = w.B if B is None else B
    heads = 2 if w.mask else 1
    J = w.offset_groups * w.K
    trunk = 2 * b * L * w.C_in * (w.K + heads * J)
    return trunk + 2 * b * L * w.C_out * (w.C_in // w.groups) * w.K


def packed_trunk_bytes(w: W.Workload) -> int:
    """The trunk's tensors counted once: x and the trunk weights read, the predicted offsets
    (and mask) written."""
    es = 4 if w.dtype == "f32" else 2
    heads = 2 if w.mask else 1
    J = w.offset_groups * w.K
    n = w.B * w.C_in * w.L_in + w.C_in * (w.K + 1) + heads * J * (w.C_in + 1)
    n += heads * w.B * J * w.L_out
    return n * es


def packed_layer_bytes(w: W.Workload) -> int:
    """The fused layer's tensors counted once: x, the trunk weights and the deformable
    weight and bias read, the output written (the predicted offsets and mask stay on chip)."""
    es = 4 if w.dtype == "f32" else 2
    heads = 2 if w.mask else 1
    J = w.offset_groups * w.K
    n = w.B * w.C_in * w.L_in + w.C_in * (w.K + 1) + heads * J * (w.C_in + 1)
    n += w.C_out * (w.C_in // w.groups) * w.K + (w.C_out if w.bias_dist is not None else 0)
    n += w.B * w.C_out * w.L_out
    return n * es


def time_oracle_packed(w: W.Workload, host: dict, target_s: float):
    """The oracle layer on the first positions of batch element 0, grown to about target_s."""
    import oracle
    L = 64
    while True:
        Ls = min(w.L_in, L)
        sl = dict(host)
        sl["x"] = host["x"][:1, :, :Ls]
        t0 = time.perf_counter()
        _, _, _ = oracle.packed_forward(*[sl[k] for k in PACKED_KEYS], w.stride, w.padding,
                                        w.dilation, w.groups, w.offset_groups,
                                        w.unconstrained)
        dt = time.perf_counter() - t0
        L_out = oracle.out_length(Ls, w.K, w.stride, w.padding, w.dilation)
        if dt > target_s / 4 or Ls >= w.L_in:
            return packed_flops(w, L_out, 1) / dt / 1e12, L_out, dt, oracle.threads()
        L = int(L * max(2.0, min(8.0, target_s / 4 / max(dt, 1e-3))))


def run_packed_pass(args, w: W.Workload, peaks: dict, want_cpu: bool):
    """One step = PackedDeformConv1d's forward of one batch: for the depthwise layer one
    kernel whose predicted offsets and mask never leave the chip, otherwise the trunk
    (predicted tensors in the workspace) and then the deformable convolution."""
    import deformable_convolution_dcn1d_b200 as dcn
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dcn.load()
    host = W.make_packed_inputs(w, seed=rank)
    d = {k: (v.to(dev) if v is not None else None) for k, v in host.items()}
    out = torch.empty((w.B, w.C_out, w.L_out), dtype=w.torch_dtype, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    pads = (w.padding, w.padding)

    def step(t, o):
        dcn.dcn1d_packed_forward(*[t[k] for k in PACKED_KEYS], w.stride, pads, w.dilation,
                                 w.groups, w.offset_groups, w.unconstrained, out=o,
                                 stream=stream)

    trunk_kernel = dcn.dcn1d_packed_trunk_kernel_name(*[d[k] for k in PACKED_KEYS[:7]],
                                                      w.stride, pads, w.dilation,
                                                      w.offset_groups)
    layer_kernel = dcn.dcn1d_packed_forward_kernel_name(*[d[k] for k in PACKED_KEYS], w.stride,
                                                        pads, w.dilation, w.groups,
                                                        w.offset_groups, w.unconstrained)
    fused = layer_kernel == "packed_fused_tcgen05"
    for _ in range(max(args.warmup, 0)):
        flush.zero_()
        step(d, out)
    torch.cuda.synchronize(dev)
    launches = dcn.dcn1d_last_launch_count()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(ws)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            step(d, out)
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
    barrier(ws)
    ms_step = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), ws) / args.steps
    # the trunk kernel's own time (the library's timing events go to the first launch)
    k_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    k_ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for e in k_starts + k_ends:
        e.record(stream)
    barrier(ws)
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.zero_()
        dcn.dcn1d_set_timing_events(k_starts[i], k_ends[i])
        step(d, out)
    torch.cuda.synchronize(dev)
    barrier(ws)
    ms_trunk = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(k_starts, k_ends)),
                              ws) / args.steps
    flops = packed_flops(w)
    value = ws * flops / (ms_step / 1e3) / 1e12

    # end to end: x and every weight from pinned host memory, the output back
    pinned = {k: (v.pin_memory() if v is not None else None) for k, v in host.items()}
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in pinned.values() if v is not None)
    d2h = out_host.numel() * out_host.element_size()

    def launch(t, o, s):
        dcn.dcn1d_packed_forward(*[t[k] for k in PACKED_KEYS], w.stride, pads, w.dilation,
                                 w.groups, w.offset_groups, w.unconstrained, out=o, stream=s)

    e_ms = pipelined_e2e(dev, pinned, out.shape, out.dtype, launch, args.steps, args.warmup,
                         ws) * args.steps
    e_value = ws * flops / (e_ms / args.steps / 1e3) / 1e12

    # roofline of the timed kernel (the fused layer, else the trunk): the slower of its
    # tensor-core time (the trunk's contraction) and its HBM time
    heads = 2 if w.mask else 1
    t_flops = 2 * w.B * w.L_out * w.C_in * (w.K + heads * w.offset_groups * w.K)
    t_bytes = packed_layer_bytes(w) if fused else packed_trunk_bytes(w)
    t_tensor = t_flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = t_bytes / (peaks["hbm_gbs"] * 1e9)
    sec = ms_trunk / 1e3
    if t_hbm >= t_tensor:
        roof = {"bound": "hbm", "achieved": t_bytes / sec / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": t_flops / sec / 1e12,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
    timed = layer_kernel if fused else trunk_kernel
    roof.update({"frac": roof["achieved"] / roof["peak"],
                 "traffic": load_traffic(timed, w), "kernel": timed,
                 "peak_source": f"measured ({peaks['source']}); the bound is the slower of "
                                f"{t_tensor * 1e6:.1f} us of tensor work and "
                                f"{t_hbm * 1e6:.1f} us of HBM traffic",
                 "algorithmic_flops": t_flops, "algorithmic_bytes": t_bytes,
                 "tensor_frac": t_flops / sec / 1e12 / peaks["bf16_tflops"],
                 "hbm_frac": t_bytes / sec / 1e9 / peaks["hbm_gbs"],
                 "launches_per_step": launches, "kernel_ms": ms_trunk,
                 "timing": "CUDA events the library records around the "
                           + ("fused layer kernel" if fused else "trunk kernel")
                           + ", per step, in a second timed run of the same K steps"})
    line = {"metric": METRIC_PACKED, "value": value, "unit": "TFLOP/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic (seeded, shapes and distributions of the named "
                                      "workload; random trunk weights)",
            "config": workload_config(w, layer_kernel, ws,
                                      l2="flushed between steps (256 MiB write outside the "
                                         "timed events)"),
            "roofline": roof, "clocks": clk.summary(),
            "e2e": {"value": e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "note": "pinned host x and weights copied in, layer forward, output "
                            "out, every step; steps pipelined over two device buffer sets "
                            "(copies in, forward and copies out on three streams)"},
            "gpu_launches": launches * args.steps}
    line["config"]["modulated"] = w.mask
    if want_cpu and ws == 1 and rank == 0:
        v, n, dt, cores = time_oracle_packed(w, host, args.cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                "sample": f"the layer on the first {n} output positions of "
                                          f"batch element 0 ({dt:.1f} s)"}
    return line if rank == 0 else None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help="one of %s, or 'all'; --pass packed takes %s"
                         % (", ".join(W.WORKLOADS), ", ".join(W.PACKED)))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--pass", dest="which", default="forward",
                    choices=["forward", "backward", "packed"],
                    help="time the forward (the default line) or the backward pass")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (small cases for profiling)")
    ap.add_argument("--dtype", default=None, choices=["f16"],
                    help="run a bf16 workload's shapes and distributions in float16 instead")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    names = list(W.WORKLOADS) if args.workload == "all" else [args.workload]
    ws, rank, local = dist_env()

    if args.which == "packed" and args.workload == DEFAULT_WORKLOAD:
        names = ["packed_modulated_bf16"]

    def pick(name):
        w = W.WORKLOADS[name] if name in W.WORKLOADS else W.PACKED[name]
        if args.dtype:
            if w.dtype != "bf16":
                raise SystemExit("--dtype f16 applies to the bf16 workloads only")
            w = dataclasses.replace(w, name=w.name.replace("bf16", args.dtype), dtype=args.dtype)
        return w.with_batch(args.batch) if args.batch else w

    if args.impl == "reference":
        line = run_reference(args, pick(names[0]))
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    peaks = load_peaks()
    try:
        for name in names:
            run = {"backward": run_backward_pass, "packed": run_packed_pass}.get(args.which,
                                                                                run_ours)
            line = run(args, pick(name), peaks, want_cpu=not args.no_cpu_baseline)
            if line is not None:
                print(json.dumps(line), flush=True)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
