"""MXFP4 expert weights on the decode path (moe_forward_mxfp4) against the
fp64 oracle on the dequantized weights.

"Mixture of Experts (MoEs) in Transformers", section From Dense to Sparse:
gpt-oss generation is bound by the bytes of its active parameters, and
native mxfp4 kernels would speed it up.  The format is the OCP Microscaling
v1.0 MXFP4 (E2M1 elements, one E8M0 scale per 32 along the reduction
dimension); the oracle dequantizes it from the specification's definition
(pinned in test_oracle.py) and evaluates the layer in fp64.  The GPU forms
each block's 32 products in f16 (exact weights, the token vector scaled by
a power of two) and the blocks' sums in float32, so the bf16 tolerance
applies; routing (bf16 router) is checked as everywhere else.
"""
import ctypes

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
import sparse_mixture_experts_19_b200 as moe_pkg
from parity_util import TOL, cap_of, check_selection, host_f64, rowwise_rel_err, to_device

CASES = [
    mi.GPTOSS.with_(name="gpt_oss_mxfp4_T1", T=1),
    mi.GPTOSS.with_(name="gpt_oss_mxfp4_T2", T=2),
    mi.GPTOSS.with_(name="gpt_oss_mxfp4_T8", T=8),  # 32 slots, the size limit
    mi.Workload("mxfp4_ragged_T7", T=7, H=352, I=160, E=24, k=4),  # 28 slots, 3 columns per CTA with a tail
    # above 32 slots: the tile path, its GEMMs converting the codes in shared memory
    mi.GPTOSS.with_(name="gpt_oss_mxfp4_T64", T=64),
    mi.Workload("mxfp4_tile_ragged", T=45, H=352, I=160, E=24, k=4),  # 180 slots, ragged tiles
    mi.Workload("mxfp4_tile_cap", T=40, H=256, I=128, E=8, k=2, capacity_factor=0.75),
    # H = I = 3072: 96 scale bytes per row, the MXFP4 GEMMs' limit
    mi.Workload("mxfp4_tile_kmax", T=40, H=3072, I=3072, E=4, k=2),
    # I / 32 above the MXFP4 GEMMs' 96 scale bytes per row: dequantized to bf16 first
    mi.Workload("mxfp4_dequant_path", T=40, H=256, I=3104, E=4, k=1),
    # more than 128 rows per expert: dequantized to bf16 first
    mi.Workload("mxfp4_dequant_rows", T=600, H=256, I=128, E=4, k=2),
    mi.Workload("mxfp4_small_cap", T=2, H=256, I=128, E=8, k=4, capacity_factor=0.5),
    mi.Workload("mxfp4_one_expert", T=8, H=128, I=96, E=1, k=1),
    mi.Workload("mxfp4_e256", T=1, H=512, I=256, E=256, k=8, zipf_s=1.1),
]


def run_mx(moe, wl, inp, mx):
    d = to_device(inp, "bf16")
    dm = {n: tuple(torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in mx[n]) for n in mx}
    cfg = moe.config(wl.T, wl.H, wl.I, wl.E, wl.k, 0, wl.capacity_factor, "bf16")
    ws = moe.mxfp4_workspace(cfg)
    y = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    dropped = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    moe.moe_forward_mxfp4(cfg, d["x"], d["router_w"], d["router_b"], *dm["w_gate"], *dm["w_up"], *dm["w_down"], y,
                          idx, counts, dropped, ws)
    assert moe.moe_get_device_status(cfg, ws) == 0
    return y, idx.cpu().numpy(), counts.cpu().numpy(), dropped.cpu().numpy()


@pytest.mark.gpu
@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_mxfp4_layer_matches_oracle(gpu_lib, wl):
    inp = mi.make_inputs(wl, router_only=True)
    mx = mi.make_mxfp4_experts(wl)
    y, idx_g, counts_g, dropped_g = run_mx(gpu_lib, wl, inp, mx)
    logits, idx_o, _ = oracle.route(inp["x"], inp["router_w"], inp["router_b"], wl.k, "bf16")
    check_selection(logits, idx_o, oracle.topk_margin(logits, wl.k), idx_g, wl.k)
    perm = oracle.permute(idx_g, wl.E, cap_of(wl))
    assert np.array_equal(counts_g, perm["counts"]) and np.array_equal(dropped_g, perm["dropped"])
    yhat = oracle.moe_tokens_mxfp4(inp["x"], mx, idx_g, oracle.weights_for(logits, idx_g), "bf16",
                                   row_of=perm["row_of"])
    err = rowwise_rel_err(host_f64(y), yhat)
    assert err <= TOL["bf16"], f"{wl.name}: row-wise relative error {err:.3e}"


@pytest.mark.gpu
@pytest.mark.parametrize("T", [2, 24], ids=["decode", "tile"])
def test_mxfp4_nan_scale_reaches_only_the_tokens_that_read_it(gpu_lib, T):
    """A scale byte of 255 (NaN) in one expert's gate rows: the tokens routed
    to that expert get NaN outputs, as in the oracle; the others do not
    (4 slots: the decode kernel; 48: the tile path's MXFP4 GEMMs)."""
    wl = mi.Workload("mxfp4_nan", T=T, H=256, I=128, E=8, k=2)
    inp = mi.make_inputs(wl, router_only=True)
    mx = mi.make_mxfp4_experts(wl)
    logits, idx_o, _ = oracle.route(inp["x"], inp["router_w"], None, wl.k, "bf16")
    e_hit = int(idx_o[0, 0])
    blocks, scales = mx["w_gate"]
    scales = scales.copy()
    scales[e_hit, 3, 0] = 255
    mx = dict(mx, w_gate=(blocks, scales))
    y, idx_g, _, _ = run_mx(gpu_lib, wl, inp, mx)
    yhat = oracle.moe_tokens_mxfp4(inp["x"], mx, idx_g, oracle.weights_for(logits, idx_g), "bf16")
    yg = host_f64(y)
    assert np.array_equal(np.isnan(yg).all(1), np.isnan(yhat).all(1))
    assert np.isnan(yg[0]).all()


def _cfg(**kw):
    base = dict(T=2, H=256, I=128, E=8, top_k=4, I_shared=0, capacity_factor=0.0, dtype="bf16")
    base.update(kw)
    return moe_pkg.config(**base)


def test_mxfp4_validates():
    lib = moe_pkg.load()
    F = 0x7f0000000000

    def call(c):
        need = lib.moe_workspace_size(ctypes.byref(c))
        return lib.moe_forward_mxfp4(ctypes.byref(c), F, F, None, F, F, F, F, F, F, F, None, None, None, F, need,
                                     None)

    assert call(_cfg(I_shared=64)) == 2 and "shared" in moe_pkg.moe_last_error()
    assert call(_cfg(H=264)) == 1 and "32" in moe_pkg.moe_last_error()
    assert call(_cfg(dtype="f32")) == 2
    assert call(_cfg(T=0)) == 0
    # 36 slots with I = 3104 (> 3072): the dequantizing path, which needs the larger workspace
    c = _cfg(T=9, I=3104)
    assert lib.moe_mxfp4_workspace_size(ctypes.byref(c)) == lib.moe_workspace_size(ctypes.byref(c)) + 3 * 8 * 256 * 3104 * 2
    assert call(c) == 3 and "moe_mxfp4_workspace_size" in moe_pkg.moe_last_error()
    # 36 slots within the MXFP4 GEMMs' limits: no extra workspace
    c = _cfg(T=9)
    assert lib.moe_mxfp4_workspace_size(ctypes.byref(c)) == lib.moe_workspace_size(ctypes.byref(c))
    # 2400 slots over 8 experts (> 128 rows each): the dequantizing path again
    c = _cfg(T=600)
    assert lib.moe_mxfp4_workspace_size(ctypes.byref(c)) == lib.moe_workspace_size(ctypes.byref(c)) + 3 * 8 * 256 * 128 * 2
    # up to 32 slots the decode kernel needs no more than moe_forward
    c = _cfg(T=8)
    assert lib.moe_mxfp4_workspace_size(ctypes.byref(c)) == lib.moe_workspace_size(ctypes.byref(c))
