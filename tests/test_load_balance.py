"""Router importance, the statistic of the load-balance penalties, on the GPU.

importance[e] = sum over tokens of the softmax over all E router scores
("2026年人工智能MoE混合专家模型入门指南", the MoE layer's load-balance loss;
"模型的“分工的艺术”：MoE技术如何提升计算效率", section 3.1).  Every router
path (tensor-core, few-token exact, float32 CUDA-core) adds it as a side
output of moe_route_importance; the oracle computes it in fp64 from its own
scores.  Tolerance: the tensor-core path scores in float32 (|error| ~ 1e-5 at
these sizes, which moves a probability by about that relative amount) and
every path sums probabilities with float32 atomic adds, so 1e-4 relative per
expert with a floor of 1e-6 T.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from parity_util import to_device

RTOL = 1e-4

CASES = [
    # tensor-core router: T*E*H > 2^26, ragged last tile, Zipf bias
    mi.Workload("imp_tc_e128", T=1000, H=1024, I=64, E=128, k=8, zipf_s=1.1),
    mi.Workload("imp_tc_e256", T=600, H=512, I=64, E=256, k=8, zipf_s=1.1),
    mi.Workload("imp_tc_e8", T=9000, H=1024, I=64, E=8, k=2),
    # tensor-core router, every expert selected (k = E)
    mi.Workload("imp_tc_dense", T=3000, H=1024, I=64, E=32, k=32),
    # few tokens: the exact cluster router, bf16 and float32
    mi.Workload("imp_decode_bf16", T=3, H=2880, I=64, E=32, k=4, zipf_s=1.1),
    mi.Workload("imp_decode_f32", T=5, H=256, I=64, E=8, k=2, dtype="f32"),
    # float32 CUDA-core router
    mi.Workload("imp_simt_f32", T=4096, H=512, I=64, E=64, k=4, dtype="f32", zipf_s=1.1),
]


def run(moe, wl, d, importance, idx, w):
    cfg = moe.config(wl.T, wl.H, wl.I, wl.E, wl.k, 0, 0.0, wl.dtype)
    ws = moe.workspace(cfg)
    moe.moe_route_importance(cfg, d["x"], d["router_w"], d["router_b"], idx, w, importance, ws)
    assert moe.moe_get_device_status(cfg, ws) == 0
    return cfg, ws


@pytest.mark.gpu
@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_importance_matches_oracle(gpu_lib, wl):
    moe = gpu_lib
    inp = mi.make_inputs(wl, router_only=True)
    d = to_device(inp, wl.dtype)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    imp = torch.zeros(wl.E, dtype=torch.float32, device="cuda")
    cfg, ws = run(moe, wl, d, imp, idx, w)
    # the selection and weights are moe_route's, bit for bit
    idx2, w2 = torch.empty_like(idx), torch.empty_like(w)
    moe.moe_route(cfg, d["x"], d["router_w"], d["router_b"], idx2, w2, ws)
    assert torch.equal(idx, idx2) and torch.equal(w.view(torch.int32), w2.view(torch.int32))

    logits, _, _ = oracle.route(inp["x"], inp["router_w"], inp["router_b"], wl.k, wl.dtype)
    ref = oracle.importance(logits)
    got = imp.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref) / np.maximum(ref, 1e-6 * wl.T)
    assert err.max() <= RTOL, (int(err.argmax()), got[err.argmax()], ref[err.argmax()])
    assert abs(got.sum() - wl.T) <= RTOL * wl.T


@pytest.mark.gpu
def test_importance_is_added_to_and_penalties_follow(gpu_lib):
    """Two calls add twice the importance; the penalties from the GPU's
    importance and counts match the oracle's."""
    moe = gpu_lib
    wl = CASES[0]
    inp = mi.make_inputs(wl, router_only=True)
    d = to_device(inp, wl.dtype)
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    once = torch.zeros(wl.E, dtype=torch.float32, device="cuda")
    twice = torch.zeros(wl.E, dtype=torch.float32, device="cuda")
    cfg, ws = run(moe, wl, d, once, idx, w)
    run(moe, wl, d, twice, idx, w)
    run(moe, wl, d, twice, idx, w)
    np.testing.assert_allclose(twice.cpu().numpy(), 2 * once.cpu().numpy(), rtol=1e-5, atol=0)

    counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(wl.E + 1, dtype=torch.int32, device="cuda")
    perm_rows = torch.empty(wl.T * wl.k, dtype=torch.int32, device="cuda")
    row_of = torch.empty(wl.T * wl.k, dtype=torch.int32, device="cuda")
    dropped = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    moe.moe_permute(cfg, idx, counts, offsets, perm_rows, row_of, dropped, ws)
    logits, idx_o, _ = oracle.route(inp["x"], inp["router_w"], inp["router_b"], wl.k, wl.dtype)
    ref = oracle.balance_losses(oracle.importance(logits), oracle.permute(idx_o, wl.E)["counts"], wl.T)
    got = moe.moe_balance_losses(once, counts, wl.T)
    for key in ("kl", "std", "switch"):
        assert abs(got[key] - ref[key]) <= 1e-3 * max(abs(ref[key]), 1e-3), (key, got[key], ref[key])
