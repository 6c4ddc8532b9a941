"""The N > 1 host logic of bench.py on CPU ranks (gloo, world size 2)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _max_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench

    # each rank's time; the job time is the slowest rank's
    ms = bench.reduce_max(10.0 + 5.0 * rank, world)
    out[rank] = (ms, bench.job_tokens_per_s(4096, 20, world, ms))
    dist.barrier()
    dist.destroy_process_group()


def test_reduce_max_and_job_throughput_two_ranks():
    world = 2
    port = free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_max_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]
    ms, tps = res[0]
    assert ms == 15.0
    assert tps == pytest.approx(4096 * 20 * 2 / 0.015)


def test_reference_arm_under_torchrun_prints_once():
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--workload", "tiny_f32", "--steps", "2", "--warmup", "1"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


# -------------------------------------------- expert-parallel decomposition
# "Mixture of Experts (MoEs) in Transformers", section Expert Parallelism:
# each device holds E/N experts, keeps only the routed pairs of its own
# experts and the partial outputs are summed by an all-reduce.  The oracle
# side of that plan: rank r evaluates the pairs whose expert lies in
# [r E/N, (r+1) E/N) (the shared expert on rank 0 only) and the all-reduce
# of the partial outputs is the single-device layer.

def _ep_worker(rank, world, port, out):
    import numpy as np
    import torch

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import moe_inputs as mi
    import oracle

    wl = mi.Workload("ep", T=40, H=48, I=32, E=8, k=2, I_shared=16, capacity_factor=0.75, dtype="bf16")
    inp = mi.make_inputs(wl)
    _, idx, w = oracle.route(inp["x"], inp["router_w"], inp["router_b"], wl.k, wl.dtype)
    row_of = oracle.permute(idx, wl.E, oracle.capacity(wl.capacity_factor, wl.T, wl.k, wl.E))["row_of"].copy()  # global capacity, token order
    e0, e1 = rank * wl.E // world, (rank + 1) * wl.E // world
    row_of[(idx < e0) | (idx >= e1)] = -1  # other ranks' experts
    shared = rank == 0
    part = oracle.moe_tokens(inp["x"], inp["w_gate"], inp["w_up"], inp["w_down"], idx, w, wl.dtype,
                             row_of=row_of, ws_gate=inp["ws_gate"] if shared else None,
                             ws_up=inp["ws_up"] if shared else None, ws_down=inp["ws_down"] if shared else None)
    y = torch.from_numpy(part)
    dist.all_reduce(y)  # the exchange step: sum of the partial outputs
    out[rank] = y.numpy()
    dist.barrier()
    dist.destroy_process_group()


def test_expert_parallel_partials_sum_to_the_layer_two_ranks():
    import numpy as np

    import moe_inputs as mi
    import oracle

    world = 2
    port = free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_ep_worker, args=(world, port, out), nprocs=world, join=True)
        ys = [out[r] for r in range(world)]
    wl = mi.Workload("ep", T=40, H=48, I=32, E=8, k=2, I_shared=16, capacity_factor=0.75, dtype="bf16")
    full = oracle.forward(wl, mi.make_inputs(wl))
    assert int(full["dropped"].sum()) > 0
    for y in ys:
        np.testing.assert_allclose(y, full["y"], rtol=0, atol=1e-12 * np.abs(full["y"]).max())
