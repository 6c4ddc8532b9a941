"""Expert parallelism: each shard holds a slice of the experts and writes a
float32 partial output; the sum of the partials is the layer.

"Mixture of Experts (MoEs) in Transformers", section Expert Parallelism: the
experts are split along their first dimension over N devices, the router's
global indices are remapped to local ones, experts a device does not hold
are left out, and the partial outputs are summed by an all-reduce.

GPU part: N shards run one after another on one device (their kernels never
wait on one another), the stacked partials go through moe_reduce_partials,
and the result is compared with moe_forward on the same inputs (and with the
oracle on the GPU's selection); the shards' counts and dropped pairs,
concatenated, equal the whole layer's bit for bit.  CPU part: argument
checks of the two entry points.
"""
import ctypes

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
import sparse_mixture_experts_19_b200 as moe_pkg
from parity_util import TOL, host_f64, oracle_given_selection, rowwise_rel_err, to_device

FAKE = 0x7f0000000000  # never dereferenced: the calls below fail validation first

CASES = [
    # tile-GEMM path, shared expert on shard 0
    mi.Workload("ep_shared", T=600, H=256, I=192, E=16, k=4, I_shared=128, zipf_s=1.1),
    # global capacity in token order, cut on every shard's experts
    mi.Workload("ep_capacity", T=1500, H=256, I=128, E=32, k=4, capacity_factor=0.9),
    # decode sizes (T*k <= 8): the decode layer with other shards' slots dropped
    mi.Workload("ep_decode", T=2, H=512, I=256, E=8, k=4, I_shared=128),
]


def shard_bounds(E, n):
    return [(r * E // n, (r + 1) * E // n) for r in range(n)]


@pytest.mark.gpu
@pytest.mark.parametrize("n", [2, 4])
@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_shards_sum_to_the_layer(gpu_lib, wl, n):
    moe = gpu_lib
    inp = mi.make_inputs(wl)
    d = to_device(inp, wl.dtype)
    cfg = moe.config(wl.T, wl.H, wl.I, wl.E, wl.k, wl.I_shared, wl.capacity_factor, wl.dtype)
    ws = moe.workspace(cfg)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    moe.moe_route(cfg, d["x"], d["router_w"], d["router_b"], idx, w, ws)
    y_ref = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    counts_ref = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    dropped_ref = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    moe.moe_forward_routed(cfg, d["x"], idx, w, None, d["w_gate"], d["w_up"], d["w_down"], d["ws_gate"],
                           d["ws_up"], d["ws_down"], y_ref, counts_ref, dropped_ref, ws)

    parts = torch.full((n, wl.T, wl.H), float("nan"), dtype=torch.float32, device="cuda")
    counts, dropped = [], []
    for r, (e0, e1) in enumerate(shard_bounds(wl.E, n)):
        ws_r = moe.workspace(cfg)
        c_r = torch.empty(e1 - e0, dtype=torch.int32, device="cuda")
        dr_r = torch.empty(e1 - e0, dtype=torch.int32, device="cuda")
        shared = (d["ws_gate"], d["ws_up"], d["ws_down"]) if r == 0 else (None, None, None)
        moe.moe_forward_expert_shard(cfg, d["x"], idx, w, e0, e1 - e0, d["w_gate"][e0:e1], d["w_up"][e0:e1],
                                     d["w_down"][e0:e1], *shared, parts[r], c_r, dr_r, ws_r)
        assert moe.moe_get_device_status(cfg, ws_r) == 0
        counts.append(c_r.cpu().numpy())
        dropped.append(dr_r.cpu().numpy())
    assert np.concatenate(counts).tolist() == counts_ref.cpu().numpy().tolist()
    assert np.concatenate(dropped).tolist() == dropped_ref.cpu().numpy().tolist()
    y_ep = torch.empty_like(y_ref)
    moe.moe_reduce_partials(cfg, parts, y_ep)
    torch.cuda.synchronize()
    # against the single-device layer (float32 sums in another order) ...
    assert rowwise_rel_err(host_f64(y_ep), host_f64(y_ref)) <= 4e-3
    # ... and against the oracle on the same selection
    logits, _, _ = oracle.route(inp["x"], inp["router_w"], inp["router_b"], wl.k, wl.dtype)
    tok = np.arange(wl.T, dtype=np.int32)
    yhat, _, _ = oracle_given_selection(wl, inp, logits, idx.cpu().numpy(), tok)
    assert rowwise_rel_err(host_f64(y_ep), yhat) <= TOL[wl.dtype]


@pytest.mark.gpu
def test_reduce_partials_sums_in_order_and_rounds_once(gpu_lib):
    moe = gpu_lib
    cfg = moe.config(3, 16, 8, 4, 2)
    g = torch.Generator(device="cuda").manual_seed(5)
    parts = torch.randn((3, 3, 16), device="cuda", generator=g)
    y = torch.empty((3, 16), dtype=torch.bfloat16, device="cuda")
    moe.moe_reduce_partials(cfg, parts, y)
    ref = ((parts[0] + parts[1]) + parts[2]).to(torch.bfloat16)
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))


def _cfg(**kw):
    base = dict(T=64, H=128, I=256, E=8, top_k=2, I_shared=0, capacity_factor=0.0, dtype="bf16")
    base.update(kw)
    return moe_pkg.config(**base)


def test_expert_shard_validates():
    lib = moe_pkg.load()
    c = _cfg()
    need = lib.moe_workspace_size(ctypes.byref(c))

    def call(begin, count, **kw):
        p = dict(x=FAKE, idx=FAKE, w=FAKE, wg=FAKE, wu=FAKE, wd=FAKE, sg=None, su=None, sd=None, y=FAKE)
        p.update(kw)
        return lib.moe_forward_expert_shard(ctypes.byref(c), p["x"], p["idx"], p["w"], begin, count, p["wg"],
                                            p["wu"], p["wd"], p["sg"], p["su"], p["sd"], p["y"], None, None, FAKE,
                                            need, None)

    assert call(6, 4) == 1 and "outside" in moe_pkg.moe_last_error()
    assert call(-1, 2) == 1
    assert call(0, 0) == 1
    assert call(0, 4, y=None) == 1 and "y_partial" in moe_pkg.moe_last_error()
    assert call(0, 4, sg=FAKE, su=FAKE, sd=FAKE) == 1  # shared weights without I_shared
    assert lib.moe_reduce_partials(ctypes.byref(c), FAKE, 0, FAKE, None) == 1
    assert lib.moe_reduce_partials(ctypes.byref(c), None, 1, FAKE, None) == 1
