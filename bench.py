#!/usr/bin/env python
"""Benchmark: fused low-rank causal dynamic short convolution, forward + backward.

One step = dsc_fwd_lowrank followed by dsc_bwd_lowrank over one batch of the chosen
workload (default: the stacked-QKV shape x [8,2048,6144], z [8,2048,32],
U [32,24576], G=1, W=4, dy ~N(0,1)).  Inputs are synthetic and seeded; x alone
(201 MB) exceeds the 126 MB L2, so no flush is inserted between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Under torchrun (N > 1) every rank runs the whole workload on its own batch (weak
scaling) and the per-step weight gradient dU is summed across ranks with NCCL, the
one exchange a data-parallel training step has for this op.  Time is measured with
CUDA events on the launching stream, bracketed by a barrier and a synchronize, and
the maximum over ranks is reported.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import dsc_inputs as di  # noqa: E402

METRIC = "achieved HBM GB/s (% of peak) and tokens/s, fused low-rank dyn-conv fwd+bwd"


def algorithmic_bytes(wl):
    """Bytes that must cross HBM once per call (each tensor counted once)."""
    e = 2 if wl.dtype == "bf16" else 4
    x = wl.tokens * wl.D * e
    z = wl.tokens * wl.R * e
    U = wl.R * wl.N * e
    fwd = x + z + U + x                                 # read x, z, U; write y
    bwd = 3 * x + z + U + wl.tokens * wl.R * 4 + wl.R * wl.N * 4   # dy, x, dx; z, U; dz, dU
    return fwd, bwd


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class Clocks:
    """SM clocks and throttle reasons during the timed region: nvidia-smi (the recipe's
    query, every 100 ms) and, since a timed region can be a few ms long, NVML read about
    every half millisecond from a thread that is initialised and polling before the region
    starts (arm) and keeps its samples only between start and stop.  The GPU is named by
    its PCI bus id, so that the sampled device is the one the CUDA device maps to whatever
    the visible-device numbering."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None
        self.thread = None
        self.nvml = []
        self.recording = False
        self.stop_flag = False
        self.max_mhz = None
        try:
            pr = torch.cuda.get_device_properties(index)
            self.bus = "%08X:%02X:%02X.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
        except Exception:
            self.bus = None

    def _poll(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = (pynvml.nvmlDeviceGetHandleByPciBusId(self.bus) if self.bus
                 else pynvml.nvmlDeviceGetHandleByIndex(self.index))
            bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ready.set()
            while not self.stop_flag:
                mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                r = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                if self.recording:
                    self.nvml.append((mhz, sorted(k for k, v in bits.items() if r & v)))
                time.sleep(0.0005)
            pynvml.nvmlShutdown()
        except Exception:
            pass
        finally:
            self.ready.set()

    def arm(self):
        """Starts the samplers ahead of the timed region; nothing is kept until start()."""
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="dsc_clocks_", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.bus or str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        import threading
        self.ready = threading.Event()
        self.thread = threading.Thread(target=self._poll, daemon=True)
        self.thread.start()
        self.ready.wait(timeout=10)

    def start(self):
        if self.thread is None:
            self.arm()
        self.recording = True

    def stop(self):
        self.recording = False
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=5)
        rows = []
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()
            with open(self.path) as f:
                for line in f:
                    parts = [s.strip() for s in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
            os.unlink(self.path)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()] + [float(m) for m, _ in self.nvml]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        if self.max_mhz:
            mx.append(float(self.max_mhz))
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = {names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"}
        for _, rs in self.nvml:
            reasons.update(rs)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows) + len(self.nvml),
                "samples_nvidia_smi": len(rows), "samples_nvml": len(self.nvml), "gpu": self.bus}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world, device):
    from dynamic_short_convolutions_causal_b200 import dp
    return dp.max_over_ranks(v, device) if world > 1 else v


# ------------------------------------------------------------------ CPU oracle baseline
def _oracle_inputs(wl):
    import numpy as np  # noqa: F401
    t = di.make(di.scaled(wl, B=1, T=min(wl.T, 2048)), "cpu", ("x", "z", "U", "dy"))
    return {k: v.to(torch.float64).numpy() for k, v in t.items()}


def _oracle_step(f, wl, L):
    """One oracle fwd + bwd on the first L tokens of one sequence; returns seconds."""
    import oracle
    t0 = time.perf_counter()
    oracle.fwd_lowrank(f["x"][:, :L], f["z"][:, :L], f["U"], wl.G, wl.W)
    oracle.bwd_lowrank(f["x"][:, :L], f["z"][:, :L], f["U"], f["dy"][:, :L], wl.G, wl.W)
    return time.perf_counter() - t0


def _oracle_sample_len(f, wl, budget_s):
    """Tokens L of one sequence whose oracle fwd + bwd takes about budget_s."""
    L0 = 16
    dt0 = _oracle_step(f, wl, L0)
    return int(max(L0, min(f["x"].shape[1], L0 * budget_s / max(dt0, 1e-6))))


def _oracle_desc(wl, L):
    return ("oracle fwd+bwd (plain C, fp64, 1 thread) on the first %d tokens of one "
            "sequence of the %s workload (D=%d, R=%d, G=%d, W=%d)" % (L, wl.name, wl.D, wl.R, wl.G, wl.W))


def oracle_sample_rate(wl, budget_s=15.0):
    """Time the CPU oracle (fwd + bwd) on a bounded sample of the workload: the first
    L tokens of one sequence, with L chosen so the run takes about `budget_s`.
    Returns (tokens/s, description, seconds)."""
    f = _oracle_inputs(wl)
    L = _oracle_sample_len(f, wl, budget_s)
    dt = _oracle_step(f, wl, L)
    return L / dt, _oracle_desc(wl, L), dt


def run_reference(args, wl, world, rank):
    """The reference arm: the CPU oracle as it stands, on host cores.  A step is one
    oracle fwd + bwd over a fixed sample of the workload (the first L tokens of one
    sequence, L sized so the whole run takes a few minutes); ms_per_step is the time of
    that sample, and the sample is named in config."""
    if rank != 0:
        return 0
    f = _oracle_inputs(wl)
    per_step = max(0.05, args.ref_budget / max(1, args.steps + args.warmup))
    L = _oracle_sample_len(f, wl, per_step)
    times = []
    for i in range(args.warmup + args.steps):
        dt = _oracle_step(f, wl, L)
        if i >= args.warmup:
            times.append(dt)
    s_step = statistics.mean(times)
    v = L / s_step
    desc = _oracle_desc(wl, L)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * s_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,s^2))",
        "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "D": wl.D, "G": wl.G, "W": wl.W,
                   "R": wl.R, "tokens_per_step": L, "sample": desc},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": desc},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm
def run_ours(args, wl, world, rank, local):
    import dynamic_short_convolutions_causal_b200 as dsc
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    wl_rank = di.scaled(wl, seed=wl.seed + 1000 * rank)
    t = di.make(wl_rank, dev, ("x", "z", "U", "dy"))
    x, z, U, dy = t["x"], t["z"], t["U"], t["dy"]
    G, W, R = wl.G, wl.W, wl.R
    y = torch.empty_like(x)
    dx = torch.empty_like(x)
    dz = torch.empty((wl.B, wl.T, R), dtype=torch.float32, device=dev)
    dU = torch.empty((R, wl.N), dtype=torch.float32, device=dev)
    ws = dsc.workspace(dsc.dsc_bwd_lowrank_workspace_bytes(wl.B, wl.T, wl.D, G, W, R, x.dtype), dev)
    path = dsc.dsc_lowrank_path(wl.B, wl.T, wl.D, G, W, R, x.dtype)
    stream = torch.cuda.current_stream(dev)
    from dynamic_short_convolutions_causal_b200 import dp

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        dsc.dsc_fwd_lowrank(x, z, U, y, G, W)
        if ev is not None:
            ev[1].record(stream)
        dsc.dsc_bwd_lowrank(x, z, U, dy, dx, dz, dU, ws, G, W)
        if ev is not None:
            ev[2].record(stream)
        if world > 1:
            dp.allreduce_weight_grad(dU)

    clocks = Clocks(local)
    clocks.arm()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ck = clocks.stop()
    ms = start.elapsed_time(end)
    ms = max_over_ranks(ms, world, dev)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    ms_step = ms / args.steps
    tokens_s = wl.tokens * world / (ms_step * 1e-3)
    fwd_b, bwd_b = algorithmic_bytes(wl)
    peak, peak_kind = read_peaks()
    gbs_step = (fwd_b + bwd_b) / (ms_step * 1e-3) / 1e9
    dom = ("dsc_bwd_lowrank", bwd_b, bwd_ms) if bwd_ms >= fwd_ms else ("dsc_fwd_lowrank", fwd_b, fwd_ms)
    achieved = dom[1] / (dom[2] * 1e-3) / 1e9
    # kernels per call: tcgen05 forward 1; tcgen05 backward 2 (U reorder with the counter
    # reset, then the main kernel, which also reduces dz and dU); CUDA-core forward 1, backward 5
    launches_fwd = 1
    launches_bwd = 2 if path & 2 else 5
    traffic = load_traffic(dom[0], wl)

    # end to end through the public API with host buffers (pinned), copies inside the region
    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(dsc, t, y, dx, dz, dU, ws, wl, world, dev, args)

    comps = None
    if world == 1 and not args.no_comparators:
        del t, x, z, U, dy, y, dx, dz, dU, ws
        torch.cuda.empty_cache()
        comps = measure_comparators(dsc, dev, peak, args)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, desc, _ = oracle_sample_rate(wl, budget_s=args.cpu_budget)
        cpu = {"value": rate, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": tokens_s, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
            "data": "synthetic (seeded N(0,s^2); no dataset)",
            "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "D": wl.D, "G": G, "W": W, "R": R,
                       "tokens_per_step_per_gpu": wl.tokens, "parallelism": "dp%d" % world,
                       "l2": "inputs larger than L2 (x is %.0f MB), no flush" % (wl.tokens * wl.D * 2 / 1e6),
                       "path": {"fwd": "tcgen05" if path & 1 else "cuda-cores",
                                "bwd": "tcgen05" if path & 2 else "cuda-cores"}},
            "hbm_gbs_step": gbs_step, "hbm_pct_of_peak_step": 100.0 * gbs_step / peak,
            "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
            "fwd_gbs": fwd_b / (fwd_ms * 1e-3) / 1e9, "bwd_gbs": bwd_b / (bwd_ms * 1e-3) / 1e9,
            "roofline": {"bound": "hbm", "kernel": dom[0], "achieved": achieved, "peak": peak,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": traffic, "algorithmic_bytes": dom[1]},
            "gpu_launches": (launches_fwd + launches_bwd) * args.steps,
            "e2e": e2e, "cpu_baseline": cpu, "clocks": ck, "comparators": comps,
        }
        print(json.dumps(line), flush=True)
    return 0


def _time_calls(fn, stream, steps, warmup=3):
    """Mean CUDA-event time (ms) of fn() on `stream`, after `warmup` untimed calls."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        fn()
    e.record(stream)
    torch.cuda.synchronize()
    return s.elapsed_time(e) / steps


def _time_graph(fn, dev, n):
    """Mean device time (ms) of fn() when n calls are captured in one CUDA graph and the
    graph is replayed (no host launch overhead between the calls)."""
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        for _ in range(3):
            fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for _ in range(n):
            fn()
    g.replay()
    torch.cuda.synchronize()
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream(dev)
    s.record(cur)
    for _ in range(3):
        g.replay()
    e.record(cur)
    torch.cuda.synchronize()
    del g
    return s.elapsed_time(e) / (3 * n)


def measure_comparators(dsc, dev, peak, args):
    """Other paths timed in the same run, each on its own workload: the in-repo static
    depthwise causal convolution (the primitive the method generalises) on the MLP-width
    shape, the fused low-rank step on the MLP-width shape, the stacked-QKV step with RoPE
    fused, the explicit-filter forward and backward on the stacked-QKV shape, and the decode
    steps (low-rank and explicit filters).
    Inputs exceed L2; times are CUDA events per call."""
    stream = torch.cuda.current_stream(dev)
    steps = max(3, min(args.steps, 10))
    out = {}

    def entry(ms, nbytes, tokens):
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"ms": ms, "algorithmic_bytes": nbytes, "gbs": gbs, "frac_of_peak": gbs / peak,
                "tokens_per_s": tokens / (ms * 1e-3)}

    names = {"static", "mlp", "rope", "explicit", "decode"}
    chosen = names if args.comparators == "all" else set(args.comparators.split(","))
    if chosen - names:
        raise SystemExit("--comparators: unknown %s (choose from %s)" % (sorted(chosen - names), sorted(names)))

    def want(name):
        return name in chosen

    if want("static"):
        # static depthwise causal conv, fwd + bwd, on the MLP-width shape
        wl = di.WORKLOADS["lowrank_mlp"]
        t = di.make(wl, dev, ("x", "dy", "ws"))
        x, dy, w = t["x"], t["dy"], t["ws"]
        y = torch.empty_like(x)
        dx = torch.empty_like(x)
        dw = torch.empty((wl.D, wl.W), dtype=torch.float32, device=dev)
        ws = dsc.workspace(dsc.dsc_static_bwd_workspace_bytes(wl.B, wl.T, wl.D, wl.W), dev)
        act = wl.tokens * wl.D * 2
        fwd_ms = _time_calls(lambda: dsc.dsc_static_fwd(x, w, y), stream, steps)
        bwd_ms = _time_calls(lambda: dsc.dsc_static_bwd(x, w, dy, dx, dw, ws), stream, steps)
        sb_f = 2 * act + wl.D * wl.W * 2
        sb_b = 3 * act + wl.D * wl.W * (2 + 4)
        out["static_conv_" + wl.name] = {
            "shape": {"B": wl.B, "T": wl.T, "D": wl.D, "W": wl.W},
            "fwd": entry(fwd_ms, sb_f, wl.tokens), "bwd": entry(bwd_ms, sb_b, wl.tokens),
            "fwd_bwd": entry(fwd_ms + bwd_ms, sb_f + sb_b, wl.tokens)}
        del t, x, dy, w, y, dx, dw, ws

    if want("mlp"):
        # fused low-rank fwd + bwd on the MLP-width shape
        t = di.make(wl, dev, ("x", "z", "U", "dy"))
        x, z, U, dy = t["x"], t["z"], t["U"], t["dy"]
        y = torch.empty_like(x)
        dx = torch.empty_like(x)
        dz = torch.empty((wl.B, wl.T, wl.R), dtype=torch.float32, device=dev)
        dU = torch.empty((wl.R, wl.N), dtype=torch.float32, device=dev)
        ws = dsc.workspace(dsc.dsc_bwd_lowrank_workspace_bytes(wl.B, wl.T, wl.D, wl.G, wl.W, wl.R), dev)
        fwd_ms = _time_calls(lambda: dsc.dsc_fwd_lowrank(x, z, U, y, wl.G, wl.W), stream, steps)
        bwd_ms = _time_calls(lambda: dsc.dsc_bwd_lowrank(x, z, U, dy, dx, dz, dU, ws, wl.G, wl.W), stream, steps)
        fb, bb = algorithmic_bytes(wl)
        out["lowrank_" + wl.name.split("_", 1)[1]] = {
            "shape": {"B": wl.B, "T": wl.T, "D": wl.D, "G": wl.G, "W": wl.W, "R": wl.R},
            "fwd": entry(fwd_ms, fb, wl.tokens), "bwd": entry(bwd_ms, bb, wl.tokens),
            "fwd_bwd": entry(fwd_ms + bwd_ms, fb + bb, wl.tokens),
            "path": dsc.dsc_lowrank_path(wl.B, wl.T, wl.D, wl.G, wl.W, wl.R)}
        del t, x, z, U, dy, y, dx, dz, dU, ws

    if want("rope"):
        # the stacked-QKV step with RoPE fused on Q and K (heads of 128 channels): the op's
        # output rotated before it is stored, and the backward from the rotated gradient
        wl = di.WORKLOADS["lowrank_qkv"]
        t = di.make(wl, dev, ("x", "z", "U", "dy"))
        x, z, U, dy = t["x"], t["z"], t["U"], t["dy"]
        dh, n_rot = 128, 2 * wl.D // 3
        inv = 10000.0 ** (-torch.arange(0, dh, 2, dtype=torch.float64, device=dev) / dh)
        th = torch.arange(wl.T, dtype=torch.float64, device=dev)[:, None] * inv[None, :]
        cs = torch.stack([torch.cos(th), torch.sin(th)], dim=-1).to(torch.float32).permute(1, 0, 2).contiguous()
        y = torch.empty_like(x)
        dx = torch.empty_like(x)
        dz = torch.empty((wl.B, wl.T, wl.R), dtype=torch.float32, device=dev)
        dU = torch.empty((wl.R, wl.N), dtype=torch.float32, device=dev)
        ws = dsc.workspace(dsc.dsc_bwd_lowrank_workspace_bytes(wl.B, wl.T, wl.D, wl.G, wl.W, wl.R), dev)
        fwd_ms = _time_calls(lambda: dsc.dsc_fwd_lowrank_rope(x, z, U, cs, y, wl.G, wl.W, dh, n_rot), stream, steps)
        bwd_ms = _time_calls(lambda: dsc.dsc_bwd_lowrank_rope(x, z, U, cs, dy, dx, dz, dU, ws, wl.G, wl.W, dh, n_rot),
                             stream, steps)
        fb, bb = algorithmic_bytes(wl)
        out["lowrank_rope_" + wl.name.split("_", 1)[1]] = {
            "shape": {"B": wl.B, "T": wl.T, "D": wl.D, "G": wl.G, "W": wl.W, "R": wl.R, "dh": dh, "n_rot": n_rot},
            "fwd": entry(fwd_ms, fb, wl.tokens), "bwd": entry(bwd_ms, bb, wl.tokens),
            "fwd_bwd": entry(fwd_ms + bwd_ms, fb + bb, wl.tokens),
            "note": "bytes exclude the 0.5 MB RoPE table; a separate rotation pass would add 4 x 134 MB"}
        del t, x, z, U, dy, y, dx, dz, dU, ws, cs

    if want("explicit"):
        # explicit-filter forward and backward on the stacked-QKV shape
        wl = di.WORKLOADS["tied_qkv"]
        t = di.make(wl, dev, ("x", "w", "dy"))
        x, w, dy = t["x"], t["w"], t["dy"]
        y = torch.empty_like(x)
        ms = _time_calls(lambda: dsc.dsc_fwd(x, w, y, wl.G), stream, steps)
        nb = 2 * wl.tokens * wl.D * 2 + wl.tokens * wl.NG * wl.W * 2
        dx = torch.empty_like(x)
        dw = torch.empty((wl.B, wl.T, wl.NG, wl.W), dtype=torch.float32, device=dev)
        ms_b = _time_calls(lambda: dsc.dsc_bwd(x, w, dy, dx, dw, wl.G), stream, steps)
        nb_b = 3 * wl.tokens * wl.D * 2 + wl.tokens * wl.NG * wl.W * (2 + 4)   # x, dy, dx; w in, dw out (fp32)
        out["explicit_" + wl.name] = {"shape": {"B": wl.B, "T": wl.T, "D": wl.D, "G": wl.G, "W": wl.W},
                                      "fwd": entry(ms, nb, wl.tokens), "bwd": entry(ms_b, nb_b, wl.tokens)}
        del t, x, w, dy, y, dx, dw

    if want("decode"):
        # decode step (one token per sequence, rolling window) on the stacked-QKV width
        wl = di.WORKLOADS["lowrank_qkv"]
        D, G, W, R, N = wl.D, wl.G, wl.W, wl.R, wl.N
        gen = torch.Generator(device=dev)
        gen.manual_seed(wl.seed)
        U = (torch.randn((R, N), generator=gen, device=dev) * R ** -0.5).to(torch.bfloat16)
        dec = {}
        for B in (1, 8, 64, 256, 512):
            x = torch.randn((B, D), generator=gen, device=dev).to(torch.bfloat16)
            z = torch.randn((B, R), generator=gen, device=dev).to(torch.bfloat16)
            st = torch.randn((B, W - 1, D), generator=gen, device=dev).to(torch.bfloat16)
            y = torch.empty_like(x)
            ms = _time_graph(lambda: dsc.dsc_decode_step_lowrank(x, z, U, st, y, G, W), dev, 100)
            nb = R * N * 2 + B * (D * 2 + R * 2 + 2 * (W - 1) * D * 2 + D * 2)
            fl = B * (2 * R * N + 2 * W * D)
            dec["B=%d" % B] = {"us": ms * 1e3, "algorithmic_bytes": nb, "gbs": nb / (ms * 1e-3) / 1e9,
                               "frac_of_hbm_peak": nb / (ms * 1e-3) / 1e9 / peak,
                               "tflops": fl / (ms * 1e-3) / 1e12, "tokens_per_s": B / (ms * 1e-3)}
        out["decode_lowrank_" + wl.name.split("_", 1)[1]] = {
            "shape": {"D": D, "G": G, "W": W, "R": R}, "per_batch": dec,
            "note": "device time per step: 100 steps captured in a CUDA graph and replayed (a "
                    "generation loop's launch pattern), inputs and window resident in HBM; from "
                    "B = 8 the step is the fused forward's tensor-core kernel with one row per "
                    "sequence (w = z U by tcgen05, window moved by TMA stores), below it a "
                    "CUDA-core kernel"}
        del U, x, z, st, y
        # explicit-filter decode step (tied filters of the tied_qkv shape: w_t [B, D/G, W])
        wle = di.WORKLOADS["tied_qkv"]
        Ge, We = wle.G, wle.W
        dec = {}
        for B in (1, 8, 64, 256, 512):
            x = torch.randn((B, D), generator=gen, device=dev).to(torch.bfloat16)
            w = (torch.randn((B, D // Ge, We), generator=gen, device=dev) * 0.5).to(torch.bfloat16)
            st = torch.randn((B, We - 1, D), generator=gen, device=dev).to(torch.bfloat16)
            y = torch.empty_like(x)
            ms = _time_graph(lambda: dsc.dsc_decode_step(x, w, st, y, Ge), dev, 100)
            nb = B * (D * 2 + (D // Ge) * We * 2 + 2 * (We - 1) * D * 2 + D * 2)
            dec["B=%d" % B] = {"us": ms * 1e3, "algorithmic_bytes": nb, "gbs": nb / (ms * 1e-3) / 1e9,
                               "frac_of_hbm_peak": nb / (ms * 1e-3) / 1e9 / peak, "tokens_per_s": B / (ms * 1e-3)}
        out["decode_explicit_" + wle.name.split("_", 1)[1]] = {
            "shape": {"D": D, "G": Ge, "W": We}, "per_batch": dec,
            "note": "as decode_lowrank_qkv, with the step's filters given (CUDA cores)"}
        del x, w, st, y
        torch.cuda.empty_cache()
    return out


def source_hash():
    """Hash of the sources the tensor-core calls are built from (their kernels, the
    headers they include, the entry points that dispatch to them, include/): a stored
    ncu traffic figure for dsc_fwd_lowrank / dsc_bwd_lowrank is reported only for the
    build it was measured on.  The CUDA-core kernels (stream.cu, simt.cu, decode.cu,
    halo.cu) are not part of those calls."""
    import glob
    import hashlib
    h = hashlib.sha256()
    pkg = os.path.join(ROOT, "dynamic_short_convolutions_causal_b200", "csrc")
    names = ["common.cuh", "tc_common.cuh", "tc_lowrank.cu", "tc_bwd.cu", "internal.h", "dsc_api.cu"]
    files = sorted([os.path.join(pkg, n) for n in names] + glob.glob(os.path.join(ROOT, "include", "*.h")))
    for p in files:
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_traffic(kernel, wl):
    """Per-call DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum over the
    call's kernels) from profiles/traffic.json, if its entry was captured on the
    current sources (same source_hash()); null otherwise."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        ent = d.get(wl.name, {}).get(kernel)
        if not ent or ent.get("source_hash") != source_hash():
            return None
        return ent["bytes_per_launch"]
    except Exception:
        return None


def measure_e2e(dsc, t, y, dx, dz, dU, ws, wl, world, dev, args):
    """The step through the public binding with every input copied in from pinned host
    memory (x, z, U, dy) and every output copied out (y, dx, dz, dU), each step.  Two
    figures: `serial` (copies, compute and copies back one after another on one stream)
    and the reported one, pipelined over two buffer sets: step i+1's inputs go in on a
    copy stream and step i-1's outputs come out on another while step i computes, as a
    training loop with a host data pipeline would run it.  Times are CUDA events; the
    pipelined region starts before the first step's copies and ends after the last
    step's outputs have landed."""
    G, W = wl.G, wl.W
    hin = [t[k].cpu().pin_memory() for k in ("x", "z", "U", "dy")]
    hout = [torch.empty(a.shape, dtype=a.dtype).pin_memory() for a in (y, dx, dz, dU)]
    h2d = sum(a.numel() * a.element_size() for a in hin)
    d2h = sum(a.numel() * a.element_size() for a in hout)
    din = [[torch.empty_like(t[k]) for k in ("x", "z", "U", "dy")] for _ in range(2)]
    dout = [[y, dx, dz, dU], [torch.empty_like(a) for a in (y, dx, dz, dU)]]
    ws2 = [ws, torch.empty_like(ws)]
    comp = torch.cuda.current_stream(dev)
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    from dynamic_short_convolutions_causal_b200 import dp

    def compute(bi):
        x, z, U, dy = din[bi]
        yy, dxx, dzz, dUU = dout[bi]
        dsc.dsc_fwd_lowrank(x, z, U, yy, G, W)
        dsc.dsc_bwd_lowrank(x, z, U, dy, dxx, dzz, dUU, ws2[bi], G, W)
        if world > 1:
            dp.allreduce_weight_grad(dUU)

    def serial_step():
        for d, h in zip(din[0], hin):
            d.copy_(h, non_blocking=True)
        compute(0)
        for h, d in zip(hout, dout[0]):
            h.copy_(d, non_blocking=True)

    def timed(fn, steps):
        torch.cuda.synchronize()
        barrier(world)
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(comp)
        fn(s, steps)
        e.record(comp)
        torch.cuda.synchronize()
        barrier(world)
        return max_over_ranks(s.elapsed_time(e) / steps, world, dev)

    def run_serial(start, steps):
        for _ in range(steps):
            serial_step()

    def run_pipelined(start, steps):
        s_in.wait_event(start)
        s_out.wait_event(start)
        freed = [None, None]      # compute of the buffer set done (inputs reusable)
        drained = [None, None]    # outputs of the buffer set copied out (outputs reusable)
        loaded = [None, None]
        for i in range(steps):
            bi = i & 1
            with torch.cuda.stream(s_in):
                if freed[bi] is not None:
                    s_in.wait_event(freed[bi])
                for d, h in zip(din[bi], hin):
                    d.copy_(h, non_blocking=True)
                loaded[bi] = torch.cuda.Event()
                loaded[bi].record(s_in)
            comp.wait_event(loaded[bi])
            if drained[bi] is not None:
                comp.wait_event(drained[bi])
            compute(bi)
            freed[bi] = torch.cuda.Event()
            freed[bi].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(freed[bi])
                for h, d in zip(hout, dout[bi]):
                    h.copy_(d, non_blocking=True)
                drained[bi] = torch.cuda.Event()
                drained[bi].record(s_out)
        for ev in drained:
            if ev is not None:
                comp.wait_event(ev)

    steps = max(2, min(args.steps, 10))
    for _ in range(max(1, args.warmup // 2)):
        serial_step()
    ms_serial = timed(run_serial, steps)
    timed(run_pipelined, 2)                  # warm-up of the copy streams
    ms = timed(run_pipelined, steps)
    return {"value": wl.tokens * world / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelined": "two buffer sets; step i+1's copies in and step i-1's copies out overlap step i",
            "serial": {"value": wl.tokens * world / (ms_serial * 1e-3), "ms_per_step": ms_serial}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="lowrank_qkv", choices=["lowrank_qkv", "lowrank_mlp"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-budget", type=float, default=120.0,
                    help="seconds of oracle work for the whole reference run (warm-up + steps)")
    ap.add_argument("--no-comparators", action="store_true")
    ap.add_argument("--comparators", default="all",
                    help="comma list of static,mlp,rope,explicit,decode (default all)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = di.WORKLOADS[args.workload]
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            return run_reference(args, wl, world, rank)
        return run_ours(args, wl, world, rank, local)
    finally:
        if world > 1 and args.impl == "ours":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
