#!/usr/bin/env python
"""Throughput of the routed MoE FFN layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--T TOKENS]

One step = one ``moe_forward`` call (router GEMM + top-k/softmax, grouping,
grouped gate/up GEMM with fused SwiGLU, grouped down GEMM with fused
weighted scatter-add, final cast) over one batch of T synthetic tokens of the
workload (default: the largest configuration, the fine-grained layer with
256 routed experts top-8 plus a shared expert, T = 16384).  Inputs are
seeded (``moe_inputs``) and resident in HBM when the timed region starts.

With N > 1 (torchrun, one process per GPU) every rank runs its own batch of
T tokens with its own copy of the weights (weak scaling: tokens are
independent, there is no data-path collective); the time is the max over
ranks and ``value`` counts the tokens of all ranks.

``--impl reference`` times the fp64 CPU oracle (the only reference this
method has) on the host cores on a bounded token sample per step; under
torchrun only rank 0 runs it.

Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s at 1 B200 and % of roofline (tensor peak or HBM GB/s)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
GATEUP_KERNELS = ("gateup_sm100", "gateup_simt", "decode_layer")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="fine_grained_e256_layer")
    ap.add_argument("--T", type=int, default=0, help="override the token count")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--stage", choices=["forward", "route", "mxfp4", "backward", "ep"], default="forward",
                    help="route: time moe_route alone (only x and the router weights are allocated); "
                         "mxfp4: moe_forward_mxfp4 at decode sizes; backward: moe_backward; "
                         "ep: each rank's expert-parallel compute on one GPU")
    ap.add_argument("--shards", type=int, default=8, help="with --stage ep: the number of expert shards")
    ap.add_argument("--importance", action="store_true",
                    help="with --stage route: also time moe_route_importance (router importance as a side output)")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every step from the host instead of replaying a CUDA graph of the K steps")
    return ap.parse_args()


def workload(args):
    import moe_inputs as mi

    if args.workload not in mi.FULL:
        raise SystemExit(f"unknown workload {args.workload}; one of {sorted(mi.FULL)}")
    wl = mi.FULL[args.workload]
    return wl.with_(T=args.T) if args.T else wl


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def config_of(wl, world: int = 1):
    """The workload as both arms report it (identical dicts)."""
    weights = (wl.E * 3 * wl.H * wl.I + 3 * wl.H * wl.I_shared) * (2 if wl.dtype == "bf16" else 4)
    return {"workload": wl.name, "T": wl.T, "H": wl.H, "I": wl.I, "E": wl.E, "top_k": wl.k,
            "I_shared": wl.I_shared, "capacity_factor": wl.capacity_factor, "zipf_s": wl.zipf_s,
            "seed": wl.seed, "parallelism": f"replicas{world}",
            "l2": "inputs larger than L2: %.2f GB of expert weights, the activated ones read every step"
                  % (weights / 1e9)}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                f = [c.strip() for c in line.split(",")]
                if len(f) >= 9 and f[1].replace(".", "").isdigit():
                    rows.append(f)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


# --------------------------------------------------------------- roofline
def layer_flops(wl) -> float:
    """Algorithmic FLOPs of the expert FFNs, 2*T*k*3*H*I (+ 2*T*3*H*I_s shared)."""
    return 2.0 * wl.T * wl.k * 3 * wl.H * wl.I + 2.0 * wl.T * 3 * wl.H * wl.I_shared


def layer_bytes(wl, active_experts: int) -> float:
    """Algorithmic bytes: weights of the activated experts + x + y + router (+ shared)."""
    elt = 2 if wl.dtype == "bf16" else 4
    b = active_experts * 3 * wl.H * wl.I * elt
    b += 2 * wl.T * wl.H * elt + wl.E * wl.H * elt
    b += 3 * wl.H * wl.I_shared * elt
    return float(b)


def traffic_for(kernel: str, wl):
    """DRAM bytes per launch from the committed ncu summary, if it is for this
    kernel, this workload and the kernel's current source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path)).get(kernel)
    if not d or d.get("workload") != wl.name or d.get("T") != wl.T:
        return None
    h = hashlib.sha256()
    for rel in d["sources"]:
        src = os.path.join(ROOT, rel)
        if not os.path.exists(src):
            return None
        h.update(open(src, "rb").read())
    if h.hexdigest() != d["sources_sha256"]:
        return None  # the kernel changed since the counters were taken
    return float(d["dram_bytes_per_launch"])


# ----------------------------------------------------------------- oracle
def oracle_tokens_per_s(wl, inp, target_s: float, seed: int = 3):
    """The fp64 CPU oracle on a bounded token sample: (tokens/s, n, seconds, threads)."""
    import moe_inputs as mi
    import oracle

    def run(n):
        tok = mi.sample_tokens(seed, wl.T, n)
        xs = inp["x"][tok]
        t0 = time.perf_counter()
        _, idx, w = oracle.route(xs, inp["router_w"], inp["router_b"], wl.k, wl.dtype)
        oracle.moe_tokens(xs, inp["w_gate"], inp["w_up"], inp["w_down"], idx, w, wl.dtype,
                          ws_gate=inp["ws_gate"], ws_up=inp["ws_up"], ws_down=inp["ws_down"])
        return time.perf_counter() - t0

    # calibrate on enough tokens to keep every OpenMP thread busy
    import oracle as _o

    nc = max(2, 2 * _o.threads())
    t1 = run(min(nc, wl.T)) / min(nc, wl.T)
    n = int(max(2, min(wl.T, target_s / max(t1, 1e-6))))
    dt = run(n)
    return n / dt, n, dt, oracle.threads()


# -------------------------------------------------------------- the arms
def reduce_max(v: float, world: int, device="cpu") -> float:
    """Max of v over the ranks of the default process group (v if world == 1)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(T: int, steps: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank ran `steps` batches of T tokens; the
    job took the slowest rank's time."""
    return T * steps * world / (ms_max / 1e3)


def dist_setup(args):
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    # the reference arm runs on rank 0's host cores alone: no process group
    if world > 1 and args.impl == "ours" and not dist.is_initialized():
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    return world, rank, local


def run_reference(args, wl, world, rank):
    """The CPU oracle as the reference arm: rank 0 only."""
    if rank != 0:
        return None
    import moe_inputs as mi

    inp = mi.make_inputs(wl)
    per_step = min(10.0, 150.0 / max(1, args.steps + args.warmup))
    import oracle

    oracle.build()
    # calibrate the sample once, then time W + K steps of that sample
    _, n, _, _ = oracle_tokens_per_s(wl, inp, per_step)
    times = []
    for s in range(args.warmup + args.steps):
        tok = mi.sample_tokens(100 + s, wl.T, n)
        xs = inp["x"][tok]
        t0 = time.perf_counter()
        _, idx, w = oracle.route(xs, inp["router_w"], inp["router_b"], wl.k, wl.dtype)
        oracle.moe_tokens(xs, inp["w_gate"], inp["w_up"], inp["w_down"], idx, w, wl.dtype,
                          ws_gate=inp["ws_gate"], ws_up=inp["ws_up"], ws_down=inp["ws_down"])
        if s >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = n * len(times) / total
    sample = f"{n} seeded tokens per step (routing + expert FFN, fp64), steps {args.steps}"
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(wl, world),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_ours(args, wl, world, rank, local):
    import numpy as np
    import torch
    import torch.distributed as dist

    import moe_inputs as mi
    import sparse_mixture_experts_19_b200 as moe
    from sparse_mixture_experts_19_b200 import build as moe_build

    moe_build.build()
    moe.load()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    inp = mi.make_inputs(wl)

    def to_dev(a):
        if a is None:
            return None
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
        return t.to(dev)

    d = {k: to_dev(v) for k, v in inp.items()}
    cfg = moe.config(wl.T, wl.H, wl.I, wl.E, wl.k, wl.I_shared, wl.capacity_factor, wl.dtype)
    ws = moe.workspace(cfg, dev)
    y = torch.empty((wl.T, wl.H), dtype=d["x"].dtype, device=dev)
    counts = torch.empty(wl.E, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(x_in, y_out=None):
        # enqueued on the current stream (the capture stream while a graph is recorded)
        moe.moe_forward(cfg, x_in, d["router_w"], d["router_b"], d["w_gate"], d["w_up"], d["w_down"],
                        d["ws_gate"], d["ws_up"], d["ws_down"], y if y_out is None else y_out, None, counts,
                        None, ws)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v: float) -> float:
        return reduce_max(v, world, dev)

    for _ in range(args.warmup):
        step(d["x"])
    torch.cuda.synchronize(dev)
    if moe.moe_get_device_status(cfg, ws) != 0:
        raise SystemExit("device check flags set during warm-up")
    active = int((counts > 0).sum().item())

    gpu_uuid = None
    try:
        gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
        if not gpu_uuid.startswith("GPU-"):
            gpu_uuid = "GPU-" + gpu_uuid
    except Exception:
        gpu_uuid = None

    # ---- timed region: device time of K steps, with no event inside the
    # steps.  The dominant kernel's own time (the grouped gate/up GEMM, or the
    # decode gate/up kernel) comes from a second run of the same K steps in
    # which only that kernel is bracketed by events, the per-kernel breakdown
    # from a third, fully traced run.  With graphs (default) the K steps are
    # captured once into a CUDA graph and a run is one replay.
    use_graph = not args.no_graph

    def run_k_steps(trace, sample_clocks, only=None):
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        graph = None
        if trace:
            moe.moe_trace_begin(64 * args.steps, only)
        if use_graph:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, capture_error_mode="thread_local"):
                for _ in range(args.steps):
                    step(d["x"])
        barrier()
        torch.cuda.synchronize(dev)
        sampler = ClockSampler(gpu_uuid) if sample_clocks else None
        if sampler:
            sampler.__enter__()
        ev0.record(stream)
        if use_graph:
            graph.replay()
        else:
            for _ in range(args.steps):
                step(d["x"])
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        if sampler:
            sampler.__exit__(None, None, None)
        tr = moe.moe_trace_end(64 * args.steps) if trace else []
        barrier()
        del graph
        return ev0.elapsed_time(ev1), tr, (sampler.summary() if sampler else None)

    ms_local, _, clk = run_k_steps(False, True)              # the timed run: no trace events
    ms = max_over_ranks(ms_local)
    # the dominant kernel alone: the decode layer kernel at decode sizes (bf16,
    # T*k <= 8), else the grouped gate/up GEMM
    dom_filter = "decode_layer" if (wl.dtype == "bf16" and wl.T * wl.k <= 8) else "gateup"
    _, trace_dom, _ = run_k_steps(True, False, dom_filter)
    _, trace, _ = run_k_steps(True, False)                   # every kernel

    # ---- end to end: pinned host x -> device, forward, y -> pinned host
    # Every step copies its x from pinned host memory and its y back, as a
    # serving loop would: the copies run on their own streams, so step i+1's
    # input copy and step i-1's output copy overlap step i's forward (x and y
    # double-buffered on the device; the ordering is kept by events).
    x_host = d["x"].cpu().pin_memory()
    y_host = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(d["x"]) for _ in range(2)]
    y_dev = [torch.empty_like(y) for _ in range(2)]

    def e2e_steps(n):
        main = torch.cuda.current_stream(dev)
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        start = torch.cuda.Event()
        start.record(main)
        s_in.wait_event(start)
        s_out.wait_event(start)
        x_ready = [torch.cuda.Event() for _ in range(2)]
        x_free = [torch.cuda.Event() for _ in range(2)]
        y_ready = [torch.cuda.Event() for _ in range(2)]
        y_free = [torch.cuda.Event() for _ in range(2)]
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(x_free[b])  # forward i-2 has read x_dev[b]
                x_dev[b].copy_(x_host, non_blocking=True)
                x_ready[b].record(s_in)
            main.wait_event(x_ready[b])
            if i >= 2:
                main.wait_event(y_free[b])  # y_dev[b] of step i-2 is on the host
            step(x_dev[b], y_dev[b])
            x_free[b].record(main)
            y_ready[b].record(main)
            with torch.cuda.stream(s_out):
                s_out.wait_event(y_ready[b])
                y_host[b].copy_(y_dev[b], non_blocking=True)
                y_free[b].record(s_out)
        end_in, end_out = torch.cuda.Event(), torch.cuda.Event()
        end_in.record(s_in)
        end_out.record(s_out)
        main.wait_event(end_in)
        main.wait_event(end_out)

    e2e_steps(2)
    torch.cuda.synchronize(dev)
    g2 = None
    if use_graph:
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2, capture_error_mode="thread_local"):
            e2e_steps(args.steps)
    barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    if use_graph:
        g2.replay()
    else:
        e2e_steps(args.steps)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1))
    del g2

    tokens = wl.T * args.steps * world
    value = job_tokens_per_s(wl.T, args.steps, world, ms)
    pk, pk_kind = peaks()

    # ---- roofline of the dominant kernel (grouped gate/up GEMM + SwiGLU)
    per_kernel = {}
    for name, t in trace:
        per_kernel.setdefault(name, []).append(t)
    dom_times = {}
    for name, t in trace_dom:
        dom_times.setdefault(name, []).append(t)
    dom = next((k for k in GATEUP_KERNELS if k in dom_times), None)
    roof = None
    if dom == "decode_layer":
        # the whole layer in one weight-streaming kernel: bound by HBM;
        # algorithmic bytes = the active experts' weights + x + y + router
        t_avg = sum(dom_times[dom]) / len(dom_times[dom]) / 1e3
        nbytes = layer_bytes(wl, active)
        achieved = nbytes / t_avg / 1e9
        roof = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "traffic": traffic_for(dom, wl),
                "peak_kind": f"{pk_kind} HBM copy", "launch_ms": t_avg * 1e3, "bytes_per_launch": nbytes}
    elif dom:
        t_avg = sum(dom_times[dom]) / len(dom_times[dom]) / 1e3
        kept = wl.T * wl.k
        if wl.capacity_factor > 0:
            kept = int(np.minimum(counts.cpu().numpy(), moe.capacity(cfg)).sum())
        flops = 2.0 * kept * 2 * wl.H * wl.I + 2.0 * wl.T * 2 * wl.H * wl.I_shared
        # the kernel's algorithmic bytes: the gate and up weights of the
        # active experts (+ shared), its A rows read and its h rows written
        elt = 2 if wl.dtype == "bf16" else 4
        gu_bytes = float(elt * (2 * wl.H * (active * wl.I + wl.I_shared)
                                + (kept + (wl.T if wl.I_shared else 0)) * wl.H
                                + kept * wl.I + wl.T * wl.I_shared))
        if gu_bytes / (pk["hbm_gbs"] * 1e9) > flops / (pk["bf16_tflops"] * 1e12):
            # few rows per expert: the launch is bound by reading the weights
            achieved = gu_bytes / t_avg / 1e9
            roof = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "frac": achieved / pk["hbm_gbs"], "traffic": traffic_for(dom, wl),
                    "peak_kind": f"{pk_kind} HBM copy", "launch_ms": t_avg * 1e3, "bytes_per_launch": gu_bytes,
                    "flops_per_launch": flops}
        else:
            achieved = flops / t_avg / 1e12
            # one launch of the kernel lasts milliseconds at most: burst peak
            peak = pk["bf16_tflops"]
            roof = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": traffic_for(dom, wl),
                    "peak_kind": f"{pk_kind} bf16 dense, burst", "launch_ms": t_avg * 1e3,
                    "flops_per_launch": flops, "bytes_per_launch": gu_bytes,
                    "frac_of_sustained": achieved / pk["bf16_tflops_sustained"]}
    F = layer_flops(wl)
    B = layer_bytes(wl, active)
    t_roof = max(F / (pk["bf16_tflops"] * 1e12), B / (pk["hbm_gbs"] * 1e9))
    t_roof_sus = max(F / (pk["bf16_tflops_sustained"] * 1e12), B / (pk["hbm_gbs"] * 1e9))
    t_step = ms / args.steps / 1e3
    # The K steps run back to back: when the SM clock sat below 90% of its
    # maximum (the power cap), the seconds-long sustained GEMM peak is the
    # attainable one; otherwise the burst peak.
    capped = bool(clk and clk.get("sm_mhz") and clk.get("sm_max_mhz")
                  and clk["sm_mhz"] < 0.9 * clk["sm_max_mhz"])

    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "config": config_of(wl, world),
        "launch": "cuda graph of the K steps" if use_graph else "host launches",
        "roofline": roof,
        "layer_roofline": {"t_roof_ms": (t_roof_sus if capped else t_roof) * 1e3,
                           "frac": (t_roof_sus if capped else t_roof) / t_step, "flops": F, "bytes": B,
                           "bound": "tensor" if F / (pk["bf16_tflops"] * 1e12) >= B / (pk["hbm_gbs"] * 1e9) else "hbm",
                           "peak_kind": f"{pk_kind} ({'bf16 sustained: SM clock under the power cap' if capped else 'bf16 burst'}, HBM copy)",
                           "frac_burst": t_roof / t_step, "frac_sustained": t_roof_sus / t_step},
        "kernels_ms_per_step_traced": {k: sum(v) / args.steps for k, v in per_kernel.items()},
        "kernels_note": ("per-kernel times from a separate, fully traced run of the K steps: every launch "
                         "is bracketed by its own event pair, so each time includes event overhead and "
                         "their sum exceeds ms_per_step; use them as shares, not as a breakdown of it"),
        "gpu_launches": len(trace),
        "e2e": {"value": tokens / (ms_e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": int(x_host.numel() * x_host.element_size()),
                "d2h_bytes_per_step": int(y_host[0].numel() * y_host[0].element_size()),
                "overlap": "copies on two side streams, x and y double-buffered"},
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, n, dt, threads = oracle_tokens_per_s(wl, inp, 12.0)
        out["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                               "sample": f"{n} seeded tokens of the workload (routing + expert FFN, fp64), {dt:.1f} s"}
    return out


def run_route_stage(args, wl):
    """moe_route alone on the workload's x and router weights: K steps, one line."""
    import numpy as np
    import torch

    import moe_inputs as mi
    import sparse_mixture_experts_19_b200 as moe
    from sparse_mixture_experts_19_b200 import build as moe_build

    moe_build.build()
    moe.load()
    inp = mi.make_inputs(wl, router_only=True)

    def to_dev(a):
        if a is None:
            return None
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
        return t.cuda()

    x, rw, rb = to_dev(inp["x"]), to_dev(inp["router_w"]), to_dev(inp["router_b"])
    cfg = moe.config(wl.T, wl.H, wl.I, wl.E, wl.k, wl.I_shared, wl.capacity_factor, wl.dtype)
    ws = moe.workspace(cfg)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    imp = torch.zeros(wl.E, dtype=torch.float32, device="cuda")

    def timed(call):
        for _ in range(args.warmup):
            call()
        torch.cuda.synchronize()
        moe.moe_trace_begin(8 * args.steps)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            call()
        e1.record()
        torch.cuda.synchronize()
        trace = moe.moe_trace_end(8 * args.steps)
        kern = {}
        for name, t in trace:
            kern.setdefault(name, []).append(t)
        return e0.elapsed_time(e1) / args.steps, {k: sum(v) / len(v) for k, v in kern.items()}

    ms, kern = timed(lambda: moe.moe_route(cfg, x, rw, rb, idx, w, ws))
    out = {"stage": "route", "config": config_of(wl), "ms_per_call": ms, "tokens_per_s": wl.T / (ms / 1e3),
           "x_bytes_per_s": wl.T * wl.H * (2 if wl.dtype == "bf16" else 4) / (ms / 1e3),
           "kernels_ms_per_call": kern}
    if args.importance:
        ms_i, kern_i = timed(lambda: moe.moe_route_importance(cfg, x, rw, rb, idx, w, imp, ws))
        out["importance"] = {"ms_per_call": ms_i, "kernels_ms_per_call": kern_i,
                             "sum_over_calls_per_T": float(imp.sum().item()) / wl.T}
    return out


def _stage_setup(wl, router_only=False):
    import numpy as np
    import torch

    import moe_inputs as mi
    import sparse_mixture_experts_19_b200 as moe
    from sparse_mixture_experts_19_b200 import build as moe_build

    moe_build.build()
    moe.load()
    inp = mi.make_inputs(wl, router_only=router_only)

    def to_dev(a):
        if a is None:
            return None
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)
        return t.cuda()

    return moe, inp, {k: to_dev(v) for k, v in inp.items()}


def _time_calls(args, call, flush_l2=False):
    """Device time of one call, averaged over K calls after W warm-up calls
    (CUDA events on the current stream).  flush_l2: before each timed call a
    write of 256 MB (twice L2) evicts what the previous call left in L2, and
    the events bracket each call alone; else nothing sits inside the K calls."""
    import torch

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    if flush_l2:
        buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for e0, e1 in ev:
            buf.add_(1)
            e0.record()
            call()
            e1.record()
        torch.cuda.synchronize()
        return sum(e0.elapsed_time(e1) for e0, e1 in ev) / args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        call()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / args.steps


def run_mxfp4_stage(args, wl):
    """moe_forward_mxfp4 (MXFP4 routed experts): one line, the layer's time
    against the HBM copy peak for the bytes it must read (the MXFP4 codes and
    scales of the active experts, x, y, router rows).  Up to 32 routed slots
    the decode kernel reads the codes themselves; above, the time includes
    dequantizing every expert to bf16 in the workspace."""
    import numpy as np
    import torch

    import moe_inputs as mi

    wl = wl.with_(I_shared=0)
    moe, inp, d = _stage_setup(wl, router_only=True)
    mx = mi.make_mxfp4_experts(wl)
    dm = {n: tuple(torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in mx[n]) for n in mx}
    cfg = moe.config(wl.T, wl.H, wl.I, wl.E, wl.k, 0, wl.capacity_factor, "bf16")
    ws = moe.mxfp4_workspace(cfg)
    y = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    call = lambda: moe.moe_forward_mxfp4(cfg, d["x"], d["router_w"], d["router_b"], *dm["w_gate"], *dm["w_up"],
                                         *dm["w_down"], y, None, counts, None, ws)
    # the active experts' codes fit in L2 at decode sizes, and every call
    # routes the same tokens: flush L2 between the timed calls
    ms = _time_calls(args, call, flush_l2=True)
    if moe.moe_get_device_status(cfg, ws) != 0:
        raise SystemExit("device check flags set")
    active = int((counts > 0).sum().item())
    # per active expert: three weight matrices of H*I E2M1 codes (half a
    # byte each) and one scale byte per 32 elements; plus x, y, router rows
    nbytes = active * 3 * wl.H * wl.I * (0.5 + 1.0 / 32) + 2 * wl.T * wl.H * 2 + wl.E * wl.H * 2
    pk, pk_kind = peaks()
    achieved = nbytes / (ms / 1e3) / 1e9
    conf = dict(config_of(wl), l2="L2 flushed before each timed call (a 256 MB write outside the events)")
    return {"stage": "mxfp4", "config": conf, "ms_per_call": ms, "tokens_per_s": wl.T / (ms / 1e3),
            "path": "decode kernel" if wl.T * wl.k <= 32 else (
                "tile path, MXFP4 GEMMs" if max(wl.H, wl.I) <= 3072 and wl.T * wl.k <= 128 * wl.E
                else "dequantized to bf16, tile GEMMs"),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / pk["hbm_gbs"], "bytes_per_launch": nbytes, "active_experts": active,
                         "peak_kind": f"{pk_kind} HBM copy"}}


def run_backward_stage(args, wl):
    """moe_backward (every gradient of the bf16 layer): one line, its time
    against the bf16 tensor peak for its GEMM flops."""
    import torch

    moe, inp, d = _stage_setup(wl)
    dy = torch.randn((wl.T, wl.H), device="cuda").to(torch.bfloat16)
    cfg = moe.config(wl.T, wl.H, wl.I, wl.E, wl.k, wl.I_shared, wl.capacity_factor, "bf16")
    ws = torch.zeros(moe.moe_backward_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    moe.moe_route(cfg, d["x"], d["router_w"], d["router_b"], idx, w, ws)
    E, H, I, Is, T = wl.E, wl.H, wl.I, wl.I_shared, wl.T
    f32 = lambda *shape: torch.empty(shape, dtype=torch.float32, device="cuda")
    g = [f32(T, H), f32(E, H), f32(E), f32(E, I, H), f32(E, I, H), f32(E, H, I)]
    g += [f32(Is, H), f32(Is, H), f32(H, Is)] if Is else [None, None, None]
    call = lambda: moe.moe_backward(cfg, d["x"], dy, idx, w, d["router_w"], d["w_gate"], d["w_up"], d["w_down"],
                                    d["ws_gate"], d["ws_up"], d["ws_down"], *g, ws=ws)
    ms = _time_calls(args, call)
    if moe.moe_get_device_status(cfg, ws) != 0:
        raise SystemExit("device check flags set")
    # per-kernel times from one more, traced call (each launch bracketed by
    # events: shares, not a breakdown of ms_per_call)
    moe.moe_trace_begin(256)
    call()
    torch.cuda.synchronize()
    kern = {}
    for name, t in moe.moe_trace_end(256):
        kern[name] = kern.get(name, 0.0) + t
    counts = torch.bincount(idx.flatten().long(), minlength=E)
    kept = int(counts.sum().item())
    if wl.capacity_factor > 0:
        kept = int(torch.clamp(counts, max=moe.capacity(cfg)).sum().item())
    # GEMM flops: recomputed gate/up (4HI), dY.W_d (2HI), dGU.W_gu (4HI),
    # dW_gate|up (4HI), dW_down (2HI) per kept row; the same for the shared
    # expert per token; the router's weight gradient 2HE per token
    flops = 16.0 * H * I * kept + 16.0 * H * Is * T + 2.0 * H * E * T
    pk, pk_kind = peaks()
    achieved = flops / (ms / 1e3) / 1e12
    return {"stage": "backward", "config": config_of(wl), "ms_per_call": ms, "tokens_per_s": T / (ms / 1e3),
            "kernels_ms_traced": kern,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / pk["bf16_tflops"], "flops_per_launch": flops,
                         "frac_of_sustained": achieved / pk["bf16_tflops_sustained"],
                         "peak_kind": f"{pk_kind} bf16 dense, burst"}}


def run_ep_stage(args, wl):
    """Expert parallelism on one GPU: the routing once, then each of the N
    ranks' compute (moe_forward_expert_shard over the whole batch with its
    E/N experts, float32 partial output) timed alone, and the reduction of
    the N partials (moe_reduce_partials).  The exchange between GPUs (an
    all-reduce of the partials) is not timed: one GPU."""
    import torch

    moe, inp, d = _stage_setup(wl)
    n = args.shards
    cfg = moe.config(wl.T, wl.H, wl.I, wl.E, wl.k, wl.I_shared, wl.capacity_factor, "bf16")
    ws = moe.workspace(cfg)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    moe.moe_route(cfg, d["x"], d["router_w"], d["router_b"], idx, w, ws)
    parts = torch.empty((n, wl.T, wl.H), dtype=torch.float32, device="cuda")
    shard_ms = []
    for r in range(n):
        e0, e1 = r * wl.E // n, (r + 1) * wl.E // n
        shared = (d["ws_gate"], d["ws_up"], d["ws_down"]) if r == 0 else (None, None, None)
        call = lambda: moe.moe_forward_expert_shard(cfg, d["x"], idx, w, e0, e1 - e0, d["w_gate"][e0:e1],
                                                    d["w_up"][e0:e1], d["w_down"][e0:e1], *shared, parts[r],
                                                    ws=ws)
        shard_ms.append(_time_calls(args, call))
        if moe.moe_get_device_status(cfg, ws) != 0:
            raise SystemExit("device check flags set")
    y = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    red_ms = _time_calls(args, lambda: moe.moe_reduce_partials(cfg, parts, y))
    # a rank's step: its shard and the reduction (the slowest rank sets it)
    step = max(shard_ms) + red_ms
    return {"stage": "ep", "config": dict(config_of(wl), parallelism=f"ep{n}"), "shards": n,
            "shard_ms": shard_ms, "reduce_ms": red_ms, "rank_step_ms_without_exchange": step,
            "tokens_per_s_per_rank_without_exchange": wl.T / (step / 1e3),
            "exchange_bytes_per_rank": n * wl.T * wl.H * 4,
            "note": "one GPU: each rank's compute timed alone; the all-reduce of the float32 partials is not timed"}


def main():
    args = parse_args()
    wl = workload(args)
    if args.stage != "forward":
        run = {"route": run_route_stage, "mxfp4": run_mxfp4_stage, "backward": run_backward_stage,
               "ep": run_ep_stage}[args.stage]
        print(json.dumps(run(args, wl)), flush=True)
        return
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        out = run_reference(args, wl, world, rank)
    else:
        out = run_ours(args, wl, world, rank, local)
    if rank == 0 and out is not None:
        print(json.dumps(out), flush=True)
    try:
        import torch.distributed as dist

        if dist.is_initialized():
            dist.destroy_process_group()
    except Exception:
        pass


if __name__ == "__main__":
    main()
