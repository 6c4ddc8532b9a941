"""Backward pass on the GPU (moe_backward) against the fp64 oracle.

The oracle's backward (oracle.moe_backward, pinned to torch autograd in
test_oracle.py) takes the GPU's own selection and routing weights, so the
comparison is of the gradient arithmetic alone.  The GPU path rounds x, dy,
the SwiGLU activations and their gradients to bf16 around float32
tensor-core products (as the forward does), so the bf16 tolerance applies,
measured per row of each gradient (normwise: max over rows of
||g - ghat||_inf / ||ghat||_inf; tokens for dx, experts for the expert
weights, the whole tensor for the router's gradients); rows (experts) whose
oracle gradient is exactly zero must be exactly zero.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from parity_util import TOL, cap_of, to_device

pytestmark = pytest.mark.gpu

CASES = [
    mi.Workload("bwd_shared_cap_zipf", T=300, H=256, I=192, E=8, k=2, I_shared=128, zipf_s=1.1,
                capacity_factor=0.9),
    mi.Workload("bwd_e64_k8", T=400, H=256, I=128, E=64, k=8),
    mi.Workload("bwd_ragged", T=257, H=136, I=200, E=5, k=3, I_shared=72),
    mi.Workload("bwd_decode_size", T=2, H=512, I=256, E=8, k=4),
]


def rel_rows(g, ghat):
    g = np.asarray(g, np.float64).reshape(ghat.shape[0], -1)
    ghat = ghat.reshape(ghat.shape[0], -1)
    den = np.abs(ghat).max(1)
    num = np.abs(g - ghat).max(1)
    zero = den == 0
    if np.any(num[zero] != 0):
        return float("inf")
    return float(np.max(num[~zero] / den[~zero])) if np.any(~zero) else 0.0


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_backward_matches_oracle(gpu_lib, wl):
    moe = gpu_lib
    inp = mi.make_inputs(wl)
    if inp["router_b"] is None:
        inp["router_b"] = np.zeros(wl.E, np.float32)
    dy_bits = mi.normal(wl.seed, 77, (wl.T, wl.H), 1.0, "bf16")
    d = to_device(dict(inp, dy=dy_bits), "bf16")
    cfg = moe.config(wl.T, wl.H, wl.I, wl.E, wl.k, wl.I_shared, wl.capacity_factor, "bf16")
    ws = torch.zeros(moe.moe_backward_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    moe.moe_route(cfg, d["x"], d["router_w"], d["router_b"], idx, w, ws)

    def f32(*shape):
        return torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")

    E, H, I, Is, T = wl.E, wl.H, wl.I, wl.I_shared, wl.T
    g = dict(dx=f32(T, H), d_router_w=f32(E, H), d_router_b=f32(E), d_w_gate=f32(E, I, H), d_w_up=f32(E, I, H),
             d_w_down=f32(E, H, I))
    if Is:
        g.update(d_ws_gate=f32(Is, H), d_ws_up=f32(Is, H), d_ws_down=f32(H, Is))
    moe.moe_backward(cfg, d["x"], d["dy"], idx, w, d["router_w"], d["w_gate"], d["w_up"], d["w_down"], d["ws_gate"],
                     d["ws_up"], d["ws_down"], g["dx"], g["d_router_w"], g["d_router_b"], g["d_w_gate"],
                     g["d_w_up"], g["d_w_down"], g.get("d_ws_gate"), g.get("d_ws_up"), g.get("d_ws_down"), ws=ws)
    assert moe.moe_get_device_status(cfg, ws) == 0

    idx_h = idx.cpu().numpy()
    logits, _, _ = oracle.route(inp["x"], inp["router_w"], inp["router_b"], wl.k, "bf16")
    w_ref = oracle.weights_for(logits, idx_h)
    row_of = oracle.permute(idx_h, E, cap_of(wl))["row_of"]
    dy64 = mi.bf16_bits_to_f32(dy_bits).astype(np.float64)
    ref = oracle.moe_backward(inp["x"], inp["router_w"], inp["w_gate"], inp["w_up"], inp["w_down"], idx_h, w_ref,
                              dy64, "bf16", row_of=row_of, ws_gate=inp["ws_gate"], ws_up=inp["ws_up"],
                              ws_down=inp["ws_down"])
    got = {n: t.cpu().numpy() for n, t in g.items()}
    # per row for dx (tokens) and the expert weights (experts); the router's
    # gradients are sums over tokens of the softmax derivative, which cancel
    # for some experts: normwise over the whole tensor
    errs = {n: (rel_rows(got[n].reshape(1, -1), ref[n].reshape(1, -1)) if n.startswith("d_router")
                else rel_rows(got[n], ref[n])) for n in got}
    print(wl.name, {n: f"{e:.2e}" for n, e in errs.items()})
    for n, e in errs.items():
        assert e <= TOL["bf16"], (n, e)
