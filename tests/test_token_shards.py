"""Token shards of one batch with a capacity limit.

Capacity is served in global token order ("MoE稀疏架构是什么？从原理到落地的系统解读",
section 三.2), so a shard keeps, for each expert, only what the earlier
shards left of the batch's capacity C.  The one exchange step is an
all-gather of every shard's per-expert counts; each shard then takes
capacity_left = max(0, C - sum of the earlier shards' counts).

CPU part (gloo, world size 2): the exchange and the capacity it yields give
exactly the oracle's kept slots for the whole batch.  GPU part: shards run
one after another through moe_forward_routed reproduce the single call.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import moe_inputs as mi
import oracle
import sparse_mixture_experts_19_b200 as moe_pkg


def cap_of(wl) -> int:
    return oracle.capacity(wl.capacity_factor, wl.T, wl.k, wl.E)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WL = mi.Workload("shards_cap", T=1200, H=256, I=192, E=8, k=2, capacity_factor=0.8)


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def kept_in_shard(idx_shard: np.ndarray, cap_left: np.ndarray) -> np.ndarray:
    """Slots of a shard kept under per-expert capacities, in slot order."""
    run = np.zeros_like(cap_left)
    kept = np.zeros(idx_shard.size, bool)
    for s, e in enumerate(idx_shard.ravel()):
        if run[e] < cap_left[e]:
            kept[s] = True
            run[e] += 1
    return kept


def _shard_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    inp = mi.make_inputs(WL, router_only=True)
    _, idx, _ = oracle.route(inp["x"], inp["router_w"], inp["router_b"], WL.k, WL.dtype)
    lo, hi = rank * WL.T // world, (rank + 1) * WL.T // world
    mine = idx[lo:hi]
    counts = torch.from_numpy(np.bincount(mine.ravel(), minlength=WL.E).astype(np.int64))
    gathered = [torch.zeros_like(counts) for _ in range(world)]
    dist.all_gather(gathered, counts)  # the exchange step
    per_shard = torch.stack(gathered).numpy()
    batch = moe_pkg.config(WL.T, WL.H, WL.I, WL.E, WL.k, 0, WL.capacity_factor, WL.dtype)
    cap_left = moe_pkg.moe_shard_capacity_left_host(batch, per_shard, rank)  # the library's C call
    out[rank] = kept_in_shard(mine, cap_left)
    dist.barrier()
    dist.destroy_process_group()


def test_shard_capacity_exchange_matches_global_order_two_ranks():
    world = 2
    port = free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
        kept = np.concatenate([out[r] for r in range(world)])
    inp = mi.make_inputs(WL, router_only=True)
    _, idx, _ = oracle.route(inp["x"], inp["router_w"], inp["router_b"], WL.k, WL.dtype)
    ref = oracle.permute(idx, WL.E, cap_of(WL))
    assert cap_of(WL) > 0 and int(ref["dropped"].sum()) > 0
    assert np.array_equal(kept, ref["row_of"].ravel() >= 0)


def test_shard_capacity_left_host_call():
    """The C call on host counts, against values worked out by hand: a batch
    of 18 tokens, 3 experts, top-1, cf 1.0 has C = 6."""
    batch = moe_pkg.config(18, 64, 64, 3, 1, 0, 1.0, "bf16")
    assert moe_pkg.capacity(batch) == 6
    counts = np.array([[5, 0, 3], [4, 2, 1], [1, 1, 9]])
    assert moe_pkg.moe_shard_capacity_left_host(batch, counts, 0).tolist() == [6, 6, 6]
    assert moe_pkg.moe_shard_capacity_left_host(batch, counts, 1).tolist() == [1, 6, 3]
    assert moe_pkg.moe_shard_capacity_left_host(batch, counts, 2).tolist() == [0, 4, 2]
    for bad in (-1, 3):
        with pytest.raises(moe_pkg.MoeError):
            moe_pkg.moe_shard_capacity_left_host(batch, counts, bad)
    with pytest.raises(moe_pkg.MoeError):  # no capacity factor: nothing to split
        moe_pkg.moe_shard_capacity_left_host(moe_pkg.config(18, 64, 64, 3, 1), counts, 0)


# ------------------------------------------------------------------ GPU


def _to_dev(inp, dtype):
    from parity_util import to_device
    return to_device(inp, dtype)


@pytest.mark.gpu
def test_shards_reproduce_the_single_call(gpu_lib):
    """Three shards run one after another (tile-GEMM path) give y, counts and
    dropped of the single call on the whole batch, bit for bit."""
    moe = gpu_lib
    wl = WL
    d = _to_dev(mi.make_inputs(wl), wl.dtype)
    cfg = moe.config(wl.T, wl.H, wl.I, wl.E, wl.k, 0, wl.capacity_factor, wl.dtype)
    ws = moe.workspace(cfg)
    ws.fill_(0)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    moe.moe_route(cfg, d["x"], d["router_w"], d["router_b"], idx, w, ws)
    y_full = torch.empty((wl.T, wl.H), dtype=d["x"].dtype, device="cuda")
    dropped_full = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    moe.moe_forward_routed(cfg, d["x"], idx, w, None, d["w_gate"], d["w_up"], d["w_down"], None, None, None,
                           y_full, None, dropped_full, ws)
    bounds = [0, 400, 800, wl.T]
    idx_h = idx.cpu().numpy()
    per_shard = np.stack([np.bincount(idx_h[a:b].ravel(), minlength=wl.E) for a, b in zip(bounds, bounds[1:])])
    per_shard_dev = torch.from_numpy(per_shard.astype(np.int32)).cuda()
    ys, dropped = [], np.zeros(wl.E, np.int64)
    for q, (a, b) in enumerate(zip(bounds, bounds[1:])):
        cfg_q = moe.config(b - a, wl.H, wl.I, wl.E, wl.k, 0, wl.capacity_factor, wl.dtype)
        ws_q = moe.workspace(cfg_q)
        ws_q.fill_(0)
        cap_left = torch.empty(wl.E, dtype=torch.int32, device="cuda")
        moe.moe_shard_capacity_left(cfg, per_shard_dev, q, cap_left)  # cfg: the whole batch
        assert cap_left.cpu().numpy().tolist() == moe.moe_shard_capacity_left_host(cfg, per_shard, q).tolist()
        y_q = torch.empty((b - a, wl.H), dtype=d["x"].dtype, device="cuda")
        counts_q = torch.empty(wl.E, dtype=torch.int32, device="cuda")
        dropped_q = torch.empty(wl.E, dtype=torch.int32, device="cuda")
        moe.moe_forward_routed(cfg_q, d["x"][a:b].contiguous(), idx[a:b].contiguous(), w[a:b].contiguous(),
                               cap_left, d["w_gate"], d["w_up"], d["w_down"], None, None, None, y_q, counts_q,
                               dropped_q, ws_q)
        assert moe.moe_get_device_status(cfg_q, ws_q) == 0
        assert counts_q.cpu().numpy().tolist() == per_shard[q].tolist()
        ys.append(y_q)
        dropped += dropped_q.cpu().numpy()
    assert dropped.tolist() == dropped_full.cpu().numpy().tolist()
    assert int(dropped.sum()) > 0
    assert torch.equal(torch.cat(ys).view(torch.int16), y_full.view(torch.int16))


@pytest.mark.gpu
def test_decode_sized_shards_follow_the_global_capacity(gpu_lib):
    """Shards of 2 tokens (T*k = 8: the decode kernels) with a capacity that
    binds across shards: each shard's dropped slots are the oracle's for the
    whole batch, and y is within tolerance of the oracle on the same
    selection."""
    from parity_util import TOL, host_f64, oracle_given_selection, rowwise_rel_err
    moe = gpu_lib
    wl = mi.Workload("shards_decode", T=6, H=264, I=200, E=4, k=4, capacity_factor=0.5, I_shared=72)
    inp = mi.make_inputs(wl)
    d = _to_dev(inp, wl.dtype)
    cfg = moe.config(wl.T, wl.H, wl.I, wl.E, wl.k, wl.I_shared, wl.capacity_factor, wl.dtype)
    ws = moe.workspace(cfg)
    ws.fill_(0)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    moe.moe_route(cfg, d["x"], d["router_w"], d["router_b"], idx, w, ws)
    idx_h = idx.cpu().numpy()
    bounds = [0, 2, 4, 6]
    per_shard = np.stack([np.bincount(idx_h[a:b].ravel(), minlength=wl.E) for a, b in zip(bounds, bounds[1:])])
    per_shard_dev = torch.from_numpy(per_shard.astype(np.int32)).cuda()
    ys, dropped = [], np.zeros(wl.E, np.int64)
    for q, (a, b) in enumerate(zip(bounds, bounds[1:])):
        cfg_q = moe.config(b - a, wl.H, wl.I, wl.E, wl.k, wl.I_shared, wl.capacity_factor, wl.dtype)
        ws_q = moe.workspace(cfg_q)
        ws_q.fill_(0)
        cap_left = torch.empty(wl.E, dtype=torch.int32, device="cuda")
        moe.moe_shard_capacity_left(cfg, per_shard_dev, q, cap_left)
        y_q = torch.empty((b - a, wl.H), dtype=d["x"].dtype, device="cuda")
        dropped_q = torch.empty(wl.E, dtype=torch.int32, device="cuda")
        moe.moe_forward_routed(cfg_q, d["x"][a:b].contiguous(), idx[a:b].contiguous(), w[a:b].contiguous(),
                               cap_left, d["w_gate"], d["w_up"], d["w_down"], d["ws_gate"], d["ws_up"],
                               d["ws_down"], y_q, None, dropped_q, ws_q)
        assert moe.moe_get_device_status(cfg_q, ws_q) == 0
        ys.append(y_q)
        dropped += dropped_q.cpu().numpy()
    ref = oracle.permute(idx_h, wl.E, cap_of(wl))
    assert dropped.tolist() == ref["dropped"].tolist() and int(dropped.sum()) > 0
    logits, _, _ = oracle.route(inp["x"], inp["router_w"], inp["router_b"], wl.k, wl.dtype)
    yhat, _, _ = oracle_given_selection(wl, inp, logits, idx_h, np.arange(wl.T, dtype=np.int32))
    assert rowwise_rel_err(host_f64(torch.cat(ys)), yhat) <= TOL[wl.dtype]
