"""Exact selection and order on every router path, on inputs built to break
approximate routers (needs a B200).

"MoE稀疏架构是什么？从原理到落地的系统解读", section 四: the router keeps the k
largest scores; equal scores go to the lower expert index (the reading this
library takes).  Three constructions, each run through the three router
paths (tensor-core for bf16 with T*E*H > 2^26, the few-token cluster router,
and the float32 CUDA-core router):

  * exact ties: every third token is x = 0, so its scores are the router
    bias exactly, and the bias repeats values across experts;
  * identical router rows: every expert has the same score for every token,
    so the selection is experts 0..k-1 in that order;
  * cancellation: the second half of each router row nearly cancels the
    first (x repeats its first half), so the float32 partial sums are large
    and the final scores small: a rescoring band sized from the final
    scores would miss experts.

topk_idx (ordered) and the grouping counts must equal the oracle's
bit-exactly, except where the oracle's scores are within (0, 1e-5) of each
other at the selection boundary or between two selected experts.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from parity_util import check_selection, to_device

pytestmark = pytest.mark.gpu

# (name, T, H, E, k, dtype): tensor-core router needs bf16 and T*E*H > 2^26
PATHS = [
    ("tensor_core_e32", 4096, 1024, 32, 4, "bf16"),
    ("tensor_core_e256", 512, 1024, 256, 8, "bf16"),
    ("cluster_few_tokens", 8, 1024, 32, 4, "bf16"),
    ("cuda_core_f32", 4096, 1024, 32, 4, "f32"),
]


def _round(a, dtype):
    """float64 values -> the layer's input bits (bf16 bits as uint16)."""
    a32 = np.ascontiguousarray(a, np.float32)
    if dtype == "f32":
        return a32
    u = a32.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16  # round to nearest even
    return u.astype(np.uint16)


def make_case(kind, T, H, E, k, dtype):
    wl = mi.Workload(f"exact_{kind}", T=T, H=H, I=64, E=E, k=k, dtype=dtype)
    inp = mi.make_inputs(wl, router_only=True)
    rng = np.random.default_rng([T, H, E, k, len(kind), int(dtype == "bf16")])
    if kind == "ties":
        x = inp["x"].copy()
        x[::3] = 0
        inp["x"] = x
        pattern = [0.5, 1.0, 1.0, -2.0, 1.0, 0.5, 0.25, 1.0]
        inp["router_b"] = np.array([pattern[i % 8] for i in range(E)], np.float32)
    elif kind == "identical_rows":
        inp["router_w"] = np.repeat(inp["router_w"][:1], E, axis=0).copy()
    elif kind == "cancellation":
        h2 = H // 2
        w1 = rng.standard_normal((E, h2)) * 64.0
        eps = rng.standard_normal((E, h2)) * 0.02
        w = np.concatenate([w1, -w1 + eps], axis=1)
        xh = rng.standard_normal((T, h2))
        x = np.concatenate([xh, xh], axis=1)
        inp["router_w"] = _round(w, dtype)
        inp["x"] = _round(x, dtype)
    else:
        raise ValueError(kind)
    return wl, inp


def route_on_gpu(moe, wl, inp):
    d = to_device(inp, wl.dtype)
    cfg = moe.config(wl.T, wl.H, wl.I, wl.E, wl.k, 0, 0.0, wl.dtype)
    ws = moe.workspace(cfg)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    moe.moe_route(cfg, d["x"], d["router_w"], d["router_b"], idx, w, ws)
    counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    outs = [torch.empty(n, dtype=torch.int32, device="cuda") for n in (wl.E + 1, wl.T * wl.k, wl.T * wl.k, wl.E)]
    moe.moe_permute(cfg, idx, counts, *outs, ws)
    assert moe.moe_get_device_status(cfg, ws) == 0
    return idx.cpu().numpy(), w.cpu().numpy(), counts.cpu().numpy()


@pytest.mark.parametrize("kind", ["ties", "identical_rows", "cancellation"])
@pytest.mark.parametrize("path", PATHS, ids=[p[0] for p in PATHS])
def test_router_selection_and_order_are_exact(gpu_lib, kind, path):
    name, T, H, E, k, dtype = path
    wl, inp = make_case(kind, T, H, E, k, dtype)
    idx_g, w_g, counts_g = route_on_gpu(gpu_lib, wl, inp)
    logits, idx_o, w_o = oracle.route(inp["x"], inp["router_w"], inp["router_b"], k, dtype)
    margin = oracle.topk_margin(logits, k)
    exempt = check_selection(logits, idx_o, margin, idx_g, k)
    if not exempt.any():
        assert np.array_equal(counts_g, np.bincount(idx_o.ravel(), minlength=E))
    assert np.array_equal(counts_g, np.bincount(idx_g.ravel(), minlength=E))
    w_ref = oracle.weights_for(logits, idx_g)
    assert np.max(np.abs(w_g - w_ref)) < 5e-5
    if kind == "ties":
        # the zero tokens: scores are the bias, ties broken to the lower index
        zero = np.arange(0, T, 3)
        assert np.all(margin[zero] == 0.0) or k == E
        assert np.array_equal(idx_g[zero], idx_o[zero])
        bias_pick = np.argsort(-inp["router_b"].astype(np.float64), kind="stable")[:k]
        assert np.all(idx_g[zero] == bias_pick)
    if kind == "identical_rows":
        assert np.all(idx_g == np.arange(k))
