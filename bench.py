"""Benchmark of the BRA forward pass (bra_forward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload stage1] [--impl ours|reference]

A step is one bra_forward call: the whole hot path (region means, affinity + top-k,
gather-attention) over one batch of the workload. Inputs are seeded synthetic data of the
workload's shape, resident in HBM before timing starts; the step rotates through enough
input/output buffer sets (copies of the batch, rolled along the image axis) that the set it
reads was evicted from L2 by the others. The K timed steps are captured as one CUDA graph
(eager launches if capture is refused) with a timing event before the first and after the
last, on the launching stream; the median of several such runs is reported. A second graph of
bra_route then bra_attend, with an event around every call, gives the per-kernel breakdown.
With N > 1 (torchrun), each rank runs its own batch (weak scaling, no data-path collective)
and the time is the max over ranks.

The headline workload (--workload, stage1 by default) gives the line's top-level fields; every
named workload is also timed the same way and reported under "per_config" (skip with
--no-per-config). Prints one JSON line on rank 0. `--impl reference` times the CPU oracle on
the host cores instead (a bounded sample of the same workload per step).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "BRA forward tokens/s on 1 B200 (device-timed) and % of roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = {"attend_gather_umma": "bi_level_routing_b200/csrc/bra_attend_umma.cu",
                  "attend_gather_mma": "bi_level_routing_b200/csrc/bra_attend_mma.cu",
                  "attend_gather_mma_heads": "bi_level_routing_b200/csrc/bra_attend_mma.cu",
                  "attend_dense_mma": "bi_level_routing_b200/csrc/bra_attend_mma.cu",
                  "attend_dense_mma_heads": "bi_level_routing_b200/csrc/bra_attend_mma.cu",
                  "attend_region_mma": "bi_level_routing_b200/csrc/bra_attend_region.cu",
                  "attend_simt": "bi_level_routing_b200/csrc/bra_attend_simt.cu",
                  "attend_backward": "bi_level_routing_b200/csrc/bra_attend_backward.cu",
                  "lepe": "bi_level_routing_b200/csrc/bra_lepe.cu",
                  "region_means": "bi_level_routing_b200/csrc/bra_route.cu",
                  "region_means_small": "bi_level_routing_b200/csrc/bra_route.cu",
                  "region_means_padded": "bi_level_routing_b200/csrc/bra_route.cu",
                  "route_tf32x3": "bi_level_routing_b200/csrc/bra_route.cu",
                  "route_tf32x3_wide": "bi_level_routing_b200/csrc/bra_route.cu",
                  "route_heads": "bi_level_routing_b200/csrc/bra_route.cu"}
# The kernels one bra_forward step launches on each named workload (the launch lists show them);
# the step's recorded DRAM traffic is their sum.
STEP_KERNELS = {"tiny_f32": ("region_means_small", "route_tf32x3", "attend_simt"),
                "stage1": ("region_means", "route_tf32x3", "attend_gather_umma"),
                "stage2": ("region_means_small", "route_tf32x3", "attend_gather_mma"),
                "stage3": ("region_means_small", "route_tf32x3", "attend_region_mma"),
                "stage4": ("attend_dense_mma",),
                "highres": ("region_means", "route_tf32x3_wide", "attend_gather_umma")}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="stage1")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="time the headline workload only")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip per-head routing, LePE, backward and auto_pad timings")
    ap.add_argument("--eager", action="store_true", help="do not capture CUDA graphs")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="target CPU time of the oracle sample")
    ap.add_argument("--cpu-seconds-per-config", type=float, default=2.0,
                    help="target CPU time of the oracle sample of each per_config workload")
    ap.add_argument("--soak-seconds", type=float, default=1.0,
                    help="identical untimed steps before the timed region, while clocks are sampled")
    ap.add_argument("--repeats", type=int, default=5, help="timed runs of K steps; the median is reported")
    ap.add_argument("--once", choices=ONCE_ROWS, default=None,
                    help="run one row of the library --reps times on --workload, untimed, and exit (for profilers)")
    ap.add_argument("--reps", type=int, default=3, help="calls made by --once")
    return ap.parse_args(argv)


ONCE_ROWS = ("forward", "route", "attend", "forward_heads", "lepe", "forward_lepe", "backward", "auto_pad")


def run_once(args):
    """Calls one row of the library a few times on a named workload, eagerly, on fresh seeded
    inputs (auto_pad: the workload cropped by two rows and columns), checks the device error word
    and prints one line. Nothing is timed: this is the command that ncu captures."""
    import torch
    import bi_level_routing_b200 as bra
    from bi_level_routing_b200.workloads import WORKLOADS, Workload, make_inputs
    w = WORKLOADS[args.workload]
    if args.once == "auto_pad":
        w = Workload(w.name + "_cropped", w.B, w.H - 2, w.W - 2, w.C, w.heads, w.n_win, w.topk, w.dtype, w.values,
                     w.seed)
    inp = make_inputs(w)
    if w.dtype == "bf16":
        q, k, v = (torch.from_numpy(inp[n + "_bits"].view(np.int16)).view(torch.bfloat16).cuda() for n in "qkv")
    else:
        q, k, v = (torch.from_numpy(inp[n]).cuda() for n in "qkv")
    rng = np.random.Generator(np.random.PCG64(5))
    wt = torch.from_numpy(rng.standard_normal((w.C, 5, 5)) * 0.2).float().cuda()
    bias = torch.from_numpy(rng.standard_normal(w.C) * 0.1).float().cuda()
    idx = bra.route(q, k, w.n_win, w.topk) if args.once in ("attend", "backward") else None
    for _ in range(max(1, args.reps)):
        if args.once == "forward":
            bra.forward(q, k, v, w.n_win, w.topk, w.heads)
        elif args.once == "route":
            bra.route(q, k, w.n_win, w.topk)
        elif args.once == "attend":
            bra.attend(q, k, v, idx, w.heads, w.n_win)
        elif args.once == "forward_heads":
            bra.forward_heads(q, k, v, w.n_win, w.topk, w.heads)
        elif args.once == "lepe":
            bra.lepe(q, wt, bias)
        elif args.once == "forward_lepe":
            bra.forward_lepe(q, k, v, w.n_win, w.topk, w.heads, wt, bias)
        elif args.once == "backward":
            bra.attend_backward(q, k, v, idx, v, w.heads, w.n_win)
        else:
            bra.forward_auto_pad(q, k, v, w.n_win, w.topk, w.heads)
    torch.cuda.synchronize()
    status = bra.check_device_error()
    print(json.dumps({"once": args.once, "workload": w.name, "reps": args.reps, "device_error": status}))
    if status != 0:
        raise SystemExit(1)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_sha(rel: str) -> str:
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current source."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        table = json.load(f)
    rec = table.get(kernel, {}).get(workload)
    if not rec or kernel not in KERNEL_SOURCES or rec.get("source_sha256") != source_sha(KERNEL_SOURCES[kernel]):
        return None
    return rec.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        return summarize_clocks(self.lines)


def summarize_clocks(lines):
    """Median SM clock, max clock and the throttle reasons seen, from nvidia-smi csv lines."""
    sm, smax, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for ln in lines:
        parts = [p.strip() for p in ln.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            smax.append(float(parts[2]))
        except ValueError:
            continue
        for name, val in zip(names, parts[5:9]):
            if val.lower() == "active":
                reasons.add(name)
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
            "samples": len(sm)}


def cpu_baseline(w, inp, seconds: float):
    """The oracle's forward pass, as it stands, on the first images of the batch (the whole batch,
    repeated, when one pass over it takes less than `seconds`)."""
    import oracle
    orc = oracle.default()
    q, k, v = inp["q"], inp["k"], inp["v"]
    t0 = time.perf_counter()
    orc.forward(q[:1], k[:1], v[:1], w.n_win, w.topk, w.heads)
    t1 = time.perf_counter() - t0
    n = int(max(1, min(w.B, math.floor(seconds / max(t1, 1e-6)))))
    reps = 1
    if n > 1:
        t0 = time.perf_counter()
        orc.forward(q[:n], k[:n], v[:n], w.n_win, w.topk, w.heads)
        t1 = time.perf_counter() - t0
    if n == w.B and t1 < seconds:
        reps = int(max(1, min(100, math.floor(seconds / max(t1, 1e-6)))))
        t0 = time.perf_counter()
        for _ in range(reps):
            orc.forward(q, k, v, w.n_win, w.topk, w.heads)
        t1 = time.perf_counter() - t0
    return {"value": reps * n * w.N / t1, "unit": UNIT, "cores": orc.max_threads(), "kind": "oracle",
            "sample": f"oracle forward (route + attend, float64) on the first {n} of {w.B} images "
                      f"({n * w.N} query tokens) x {reps}, {t1:.2f} s"}


def run_reference(args, w, rank):
    """Reference arm: the CPU oracle timed on the host cores, rank 0 only."""
    if rank != 0:
        return
    from bi_level_routing_b200.workloads import make_inputs
    import oracle
    sample = w.with_(B=1)
    inp = make_inputs(sample)
    orc = oracle.default()
    for _ in range(args.warmup):
        orc.forward(inp["q"], inp["k"], inp["v"], w.n_win, w.topk, w.heads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        orc.forward(inp["q"], inp["k"], inp["v"], w.n_win, w.topk, w.heads)
    dt = time.perf_counter() - t0
    value = args.steps * sample.N / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": {**w.describe(), "sample_per_step": f"1 of {w.B} images ({sample.N} query tokens)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": orc.max_threads(), "kind": "oracle",
                             "sample": f"1 image of {w.name} per step, {args.steps} steps"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def step_roofline_us(w, pk) -> float:
    """max(unique q/k/v/out bytes at HBM bandwidth, routed attention flops at the bf16 peak)."""
    return max(w.unique_bytes() / (float(pk["hbm_gbs"]) * 1e9),
               w.attention_flops() / (float(pk["bf16_tflops"]) * 1e12)) * 1e6


def step_traffic(workload: str):
    """DRAM bytes of one step: the recorded per-launch traffic of each kernel the step launches,
    summed, if every one was taken on the current source; else None."""
    parts = [recorded_traffic(k, workload) for k in STEP_KERNELS.get(workload, ())]
    return float(sum(parts)) if parts and all(p is not None for p in parts) else None


def roofline_record(w, pk, pk_kind, step_us, kernel, kernel_us, route_us, breakdown_us):
    """The step against its roofline (frac) and the dominant kernel's own figures (kernel_*)."""
    hbm = float(pk["hbm_gbs"])
    roof_us = step_roofline_us(w, pk)
    achieved = w.unique_bytes() / (step_us * 1e-6) / 1e9
    kernel_achieved = w.unique_bytes() / (kernel_us * 1e-6) / 1e9
    return {"bound": "hbm", "scope": "bra_forward step (every kernel of the call)",
            "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
            "traffic": step_traffic(w.name),
            "peak_source": f"{pk_kind} hbm_gbs (MEASURED_PEAKS.json)" if pk_kind == "measured" else "fallback",
            "algorithmic_bytes_per_step": w.unique_bytes(), "step_roofline_us": roof_us, "step_us": step_us,
            "step_frac_vs_8tbs": (w.unique_bytes() / 8e12 * 1e6) / step_us,
            "dominant_kernel": {"name": kernel, "mean_launch_us": kernel_us, "achieved": kernel_achieved,
                                "unit": "GB/s", "kernel_frac": kernel_achieved / hbm,
                                "algorithmic_bytes_per_launch": w.unique_bytes(),
                                "traffic": recorded_traffic(kernel, w.name)},
            "route_kernels_mean_us": route_us, "breakdown_us_per_step": breakdown_us}


def measure(w, args, dev, world, rank, with_warm=True):
    """Times K steps of bra_forward on workload w (L2-cold rotation; one graph per run, median of
    the runs), the breakdown of route / attend, and clocks during a soak around the runs."""
    import torch
    import torch.distributed as dist
    import bi_level_routing_b200 as bra
    from bi_level_routing_b200.workloads import make_inputs

    inp = make_inputs(w, seed=w.seed + 1000 * rank)
    if w.dtype == "bf16":
        host = [torch.from_numpy(inp[n + "_bits"].view(np.int16)).view(torch.bfloat16) for n in "qkv"]
    else:
        host = [torch.from_numpy(inp[n]) for n in "qkv"]
    base = [t.to(dev) for t in host]
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2**20))
    set_bytes = w.unique_bytes() + w.B * w.R * w.topk * 4
    nsets = max(2, math.ceil(2 * l2 / set_bytes) + 1)
    sets = []
    for i in range(nsets):
        q, k, v = (torch.roll(t, shifts=i, dims=0).contiguous() for t in base)
        out = torch.empty_like(q)
        idx = torch.empty((w.B, w.R, w.topk), dtype=torch.int32, device=dev)
        sets.append((q, k, v, out, idx))
    del base
    torch.cuda.synchronize()

    def route(s):
        bra.route(s[0], s[1], w.n_win, w.topk, idx=s[4])

    def attend(s):
        bra.attend(s[0], s[1], s[2], s[4], w.heads, w.n_win, out=s[3])

    def forward(s):
        bra.forward(s[0], s[1], s[2], w.n_win, w.topk, w.heads, out=s[3], idx=s[4])

    # eager warm-up (also initialises the library's per-device state before any capture)
    for i in range(max(3, args.warmup)):
        forward(sets[i % nsets])
        route(sets[i % nsets])
        attend(sets[i % nsets])
    torch.cuda.synchronize()

    # The timed region: K steps of bra_forward captured as ONE CUDA graph with a timing event
    # (an external event-record node) before the first and after the last, so that host launch
    # overhead does not pace the GPU and consecutive kernels keep their programmatic
    # (overlapping) launches; eager launches if capture is refused. A second graph of K steps of
    # bra_route then bra_attend, with an event around every call, gives the breakdown.
    K = args.steps
    ev_start = torch.cuda.Event(enable_timing=True, external=True)
    ev_stop = torch.cuda.Event(enable_timing=True, external=True)
    ev_route = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(K)]
    ev_attend = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(K)]
    ev_end = torch.cuda.Event(enable_timing=True, external=True)

    def record_steps():
        ev_start.record()
        for i in range(K):
            forward(sets[i % nsets])
        ev_stop.record()

    def record_breakdown():
        for i in range(K):
            s = sets[i % nsets]
            ev_route[i].record()
            route(s)
            ev_attend[i].record()
            attend(s)
        ev_end.record()

    launch = "cuda_graph (all K steps in one graph)"
    graph = graph_bd = None
    if not args.eager:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                record_steps()
            graph_bd = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph_bd):
                record_breakdown()
        except Exception as e:  # capture refused: time eager launches
            graph = graph_bd = None
            launch = f"eager (graph capture failed: {type(e).__name__}: {e})"
            torch.cuda.synchronize()
    if graph is None and launch.startswith("cuda_graph"):
        launch = "eager"
    run_steps = graph.replay if graph is not None else record_steps
    run_breakdown = graph_bd.replay if graph_bd is not None else record_breakdown

    run_steps()  # untimed: the first replay also uploads the graph
    run_breakdown()
    torch.cuda.synchronize()

    sampler = ClockSampler(dev.index)
    with sampler:
        t_soak = time.perf_counter()
        while time.perf_counter() - t_soak < args.soak_seconds:
            run_steps()
            torch.cuda.synchronize()
        runs = []
        for _ in range(max(1, args.repeats)):
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            run_steps()  # K timed steps
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            runs.append(ev_start.elapsed_time(ev_stop))
        total_ms = sorted(runs)[len(runs) // 2]  # the median run
        run_breakdown()
        torch.cuda.synchronize()
        attend_ms = [ev_attend[i].elapsed_time(ev_route[i + 1] if i + 1 < K else ev_end) for i in range(K)]
        route_ms = [ev_route[i].elapsed_time(ev_attend[i]) for i in range(K)]
        breakdown_ms = ev_route[0].elapsed_time(ev_end)
        t_tail = time.perf_counter()
        while time.perf_counter() - t_tail < min(0.5, args.soak_seconds):
            run_steps()
            torch.cuda.synchronize()

    if world > 1:
        t = torch.tensor([total_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())

    warm = None
    if with_warm and graph is not None:
        ev_w0 = torch.cuda.Event(enable_timing=True, external=True)
        ev_w1 = torch.cuda.Event(enable_timing=True, external=True)
        try:
            gw = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gw):
                ev_w0.record()
                for _ in range(K):
                    forward(sets[0])
                ev_w1.record()
            gw.replay()
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            gw.replay()
            torch.cuda.synchronize()
            warm_ms = ev_w0.elapsed_time(ev_w1)
            if world > 1:
                t = torch.tensor([warm_ms], device=dev, dtype=torch.float64)
                dist.all_reduce(t, op=dist.ReduceOp.MAX)
                warm_ms = float(t.item())
            warm = {"value": w.tokens * world * K / (warm_ms / 1e3), "unit": UNIT, "ms_per_step": warm_ms / K,
                    "note": "secondary: one buffer set for every step, inputs warm in L2"}
            del gw
        except Exception as e:  # capture refused: no warm number
            warm = {"unavailable": f"{type(e).__name__}: {e}"}
            torch.cuda.synchronize()

    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    kernel = "attend_" + str(bra.selected_attend_kernel(w.B, w.H, w.W, w.C, w.heads, w.n_win, w.topk, dt))
    res = {"total_ms": total_ms, "ms_per_step": total_ms / K, "repeat_ms_per_step": [r / K for r in runs],
           "attend_us": statistics.mean(attend_ms) * 1e3, "route_us": statistics.mean(route_ms) * 1e3,
           "breakdown_us": breakdown_ms / K * 1e3, "kernel": kernel, "launch": launch, "warm": warm,
           "clocks": sampler.summary(), "nsets": nsets, "set_bytes": set_bytes, "l2": l2,
           "launches_per_step": bra.kernels_per_call("bra_forward", w.B, w.H, w.W, w.C, w.heads, w.n_win, w.topk, dt),
           "host": host, "inp": inp}
    del graph, graph_bd, sets
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def e2e_record(w, host, dev, world, K):
    """bra_forward_host on pinned host buffers: copies in and out inside the timed region."""
    import torch
    import torch.distributed as dist
    import bi_level_routing_b200 as bra
    hq, hk, hv = (t.pin_memory() for t in host)
    hout = torch.empty_like(hq).pin_memory()
    hidx = torch.empty((w.B, w.R, w.topk), dtype=torch.int32).pin_memory()
    for _ in range(2):
        bra.forward_host(hq, hk, hv, w.n_win, w.topk, w.heads, out=hout, idx=hidx)
    ke = max(3, min(20, K))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(ke):
        bra.forward_host(hq, hk, hv, w.n_win, w.topk, w.heads, out=hout, idx=hidx)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([e2e_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    return {"value": w.tokens * world * ke / (e2e_ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": 3 * w.B * w.N * w.C * w.elem_bytes,
            "d2h_bytes_per_step": w.B * w.N * w.C * w.elem_bytes + w.B * w.R * w.topk * 4,
            "steps": ke, "entry_point": "bra_forward_host"}


def time_steps(step, nsteps_sets, K, repeats, world, dev):
    """Median ms per step of K steps (step(i) works on rotation set i % nsets), captured as one
    CUDA graph with timing events around it; eager if capture is refused."""
    import torch
    import torch.distributed as dist
    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True, external=True)
    e1 = torch.cuda.Event(enable_timing=True, external=True)

    def record():
        e0.record()
        for i in range(K):
            step(i)
        e1.record()

    g = None
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            record()
        run = g.replay
    except Exception:  # capture refused: eager
        g = None
        torch.cuda.synchronize()
        run = record
    run()
    torch.cuda.synchronize()
    ts = []
    for _ in range(max(1, repeats)):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        run()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) / K)
    ms = sorted(ts)[len(ts) // 2]
    if world > 1:
        t = torch.tensor([ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    del g
    return ms


def measure_extras(args, dev, world, rank, pk, pk_kind):
    """The rows after the forward pass, each timed like the headline: per-head routing + attention,
    the LePE epilogue (alone and after the forward pass), the backward pass and auto_pad."""
    import torch
    import bi_level_routing_b200 as bra
    from bi_level_routing_b200.workloads import WORKLOADS, Workload, make_inputs
    hbm = float(pk["hbm_gbs"])
    K, reps = args.steps, args.repeats
    l2 = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 * 2**20))

    def tensors(w, seed_shift=0):
        inp = make_inputs(w, seed=w.seed + 1000 * rank + seed_shift)
        if w.dtype == "bf16":
            return [torch.from_numpy(inp[n + "_bits"].view(np.int16)).view(torch.bfloat16).to(dev) for n in "qkv"]
        return [torch.from_numpy(inp[n]).to(dev) for n in "qkv"]

    def rotation(w, per_set_bytes, make_set):
        base = tensors(w)
        nsets = max(2, math.ceil(2 * l2 / per_set_bytes) + 1)
        return [make_set([torch.roll(t, shifts=i, dims=0).contiguous() for t in base]) for i in range(nsets)]

    def record(name, w, ms, algo_bytes, note):
        achieved = algo_bytes / (ms * 1e-3) / 1e9
        return {"value": w.tokens * world / (ms * 1e-3), "unit": UNIT, "step_us": ms * 1e3,
                "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                             "algorithmic_bytes_per_step": algo_bytes,
                             "peak_source": f"{pk_kind} hbm_gbs (MEASURED_PEAKS.json)"},
                "config": w.describe(), "what": note}

    out = {}
    e = lambda w: w.elem_bytes
    # per-head routing: bra_forward_heads
    for name in ("stage1", "stage2", "stage3"):
        w = WORKLOADS[name]
        R = w.R
        sets = rotation(w, w.unique_bytes(), lambda t: (*t, torch.empty_like(t[0]),
                        torch.empty((w.B, w.heads, R, w.topk), dtype=torch.int32, device=dev)))
        step = lambda i: bra.forward_heads(*sets[i % len(sets)][:3], w.n_win, w.topk, w.heads,
                                           out=sets[i % len(sets)][3], idx=sets[i % len(sets)][4])
        ms = time_steps(step, len(sets), K, reps, world, dev)
        out[f"per_head_routing/{name}"] = record(name, w, ms, w.unique_bytes(),
                                                 "bra_forward_heads: per-head means, affinity and top-k, then "
                                                 "attention with each head's own routed regions")
        del sets
    # LePE: the epilogue alone, and bra_forward_lepe
    w = WORKLOADS["stage1"]
    rng = np.random.Generator(np.random.PCG64(5))
    wt = torch.from_numpy(rng.standard_normal((w.C, 5, 5)) * 0.2).float().to(dev)
    bias = torch.from_numpy(rng.standard_normal(w.C) * 0.1).float().to(dev)
    sets = rotation(w, 2 * w.B * w.N * w.C * e(w), lambda t: (t[0], torch.empty_like(t[0])))
    ms = time_steps(lambda i: bra.lepe(sets[i % len(sets)][0], wt, bias, out=sets[i % len(sets)][1]), len(sets), K,
                    reps, world, dev)
    out["lepe/stage1"] = record("lepe", w, ms, 2 * w.B * w.N * w.C * e(w), "bra_lepe: x + 5x5 depthwise conv + bias")
    del sets
    sets = rotation(w, 5 * w.B * w.N * w.C * e(w), lambda t: (*t, torch.empty_like(t[0]), torch.empty_like(t[0]),
                    torch.empty((w.B, w.R, w.topk), dtype=torch.int32, device=dev)))
    ms = time_steps(lambda i: bra.forward_lepe(*sets[i % len(sets)][:3], w.n_win, w.topk, w.heads, wt, bias,
                                               attn=sets[i % len(sets)][3], out=sets[i % len(sets)][4],
                                               idx=sets[i % len(sets)][5]), len(sets), K, reps, world, dev)
    out["forward_lepe/stage1"] = record("forward_lepe", w, ms, 5 * w.B * w.N * w.C * e(w),
                                        "bra_forward_lepe: routing, attention into attn, LePE epilogue into out")
    del sets
    # backward with the index fixed
    w = WORKLOADS["stage1"]
    per = (4 * e(w) + 12) * w.B * w.N * w.C

    def back_set(t):
        q, k, v = t
        idx = torch.empty((w.B, w.R, w.topk), dtype=torch.int32, device=dev)
        bra.route(q, k, w.n_win, w.topk, idx=idx)
        f32 = lambda: torch.empty((w.B, w.H, w.W, w.C), dtype=torch.float32, device=dev)
        return (q, k, v, idx, torch.flip(v, dims=[0]).contiguous(), f32(), f32(), f32())

    sets = rotation(w, per, back_set)
    ms = time_steps(lambda i: bra.attend_backward(*sets[i % len(sets)][:5], w.heads, w.n_win,
                                                  dq=sets[i % len(sets)][5], dk=sets[i % len(sets)][6],
                                                  dv=sets[i % len(sets)][7]), len(sets), K, reps, world, dev)
    out["backward/stage1"] = record("backward", w, ms, per, "bra_attend_backward: dq, dk, dv (fp32) of the token "
                                    "attention with idx fixed; bytes = q, k, v, dout read + dq, dk, dv written")
    del sets
    # auto_pad: the stage-1 shape at 54 x 54 (padded to 56 x 56 for the 7 x 7 region grid)
    w = Workload("stage1_54x54", 64, 54, 54, 64, 2, 7, 1, "bf16", "region_offset", 20267)
    sets = rotation(w, w.unique_bytes(), lambda t: (*t, torch.empty_like(t[0]),
                    torch.empty((w.B, w.R, w.topk), dtype=torch.int32, device=dev)))
    ms = time_steps(lambda i: bra.forward_auto_pad(*sets[i % len(sets)][:3], w.n_win, w.topk, w.heads,
                                                   out=sets[i % len(sets)][3], idx=sets[i % len(sets)][4]),
                    len(sets), K, reps, world, dev)
    out["auto_pad/stage1_54x54"] = record("auto_pad", w, ms, w.unique_bytes(),
                                          "bra_forward_auto_pad on 54 x 54 (zero padding to 56 x 56 read in place)")
    del sets
    torch.cuda.empty_cache()
    return out


def main(argv=None):
    args = parse_args(argv)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    from bi_level_routing_b200.workloads import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.once:
        run_once(args)
        return
    if args.impl == "reference":
        run_reference(args, w, rank)
        return

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    pk, pk_kind = peaks()
    K = args.steps
    m = measure(w, args, dev, world, rank)
    tokens = w.tokens * world
    value = tokens * K / (m["total_ms"] / 1e3)
    step_us = m["ms_per_step"] * 1e3
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic",
            "config": {**w.describe(), "l2": f"rotating {m['nsets']} buffer sets of {m['set_bytes'] / 1e6:.1f} MB "
                                             f"(> 2x the {m['l2'] / 2**20:.0f} MiB L2)",
                       "launch": m["launch"], "parallelism": f"dp{world} (images split, no collective)"},
            "roofline": roofline_record(w, pk, pk_kind, step_us, m["kernel"], m["attend_us"], m["route_us"],
                                        m["breakdown_us"]),
            "gpu_launches": K * m["launches_per_step"],
            "clocks": m["clocks"],
            "repeats": {"runs": len(m["repeat_ms_per_step"]), "ms_per_step": m["repeat_ms_per_step"],
                        "reported": "median run"}}
    if m["warm"] is not None:
        line["warm_l2"] = m["warm"]
    if not args.no_e2e:
        line["e2e"] = e2e_record(w, m["host"], dev, world, K)
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, m["inp"], args.cpu_seconds)

    # ---- every named workload, timed the same way (the headline's own entry repeats its numbers)
    if not args.no_per_config:
        per = {}
        for name, wc in WORKLOADS.items():
            mc = m if name == w.name else measure(wc, args, dev, world, rank, with_warm=False)
            sus = mc["ms_per_step"] * 1e3
            roof = roofline_record(wc, pk, pk_kind, sus, mc["kernel"], mc["attend_us"], mc["route_us"],
                                   mc["breakdown_us"])
            entry = {"value": wc.tokens * world / (sus * 1e-6), "unit": UNIT, "step_us": sus,
                     "step_roofline_us": roof["step_roofline_us"], "step_frac": roof["frac"],
                     "dominant_kernel": roof["dominant_kernel"], "route_us": mc["route_us"],
                     "breakdown_us_per_step": mc["breakdown_us"], "gpu_launches_per_step": mc["launches_per_step"],
                     "dtype": wc.dtype, "clocks": mc["clocks"], "config": wc.describe()}
            if rank == 0 and not args.no_cpu_baseline:
                entry["cpu_baseline"] = (line["cpu_baseline"] if name == w.name
                                         else cpu_baseline(wc, mc["inp"], args.cpu_seconds_per_config))
            per[name] = entry
            if mc is not m:
                del mc
        line["per_config"] = per

    if not args.no_extras:
        line["extras"] = measure_extras(args, dev, world, rank, pk, pk_kind)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
