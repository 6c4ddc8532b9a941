"""Pins of the CPU oracle against things other than itself (CPU only).

Each test pins one step of the method to an independent fact:
  * library routines: transformers' eager MoE modules (the gpt-oss top-k
    router with bias and softmax over the selected logits; the Mixtral packed
    experts), numpy / torch float64 matmuls;
  * closed forms: the two-way softmax is the logistic function; k = 1 gives
    weight 1; bias-only scores with hand-worked selections and weights;
  * special cases: top_k = E is the dense softmax mixture; E = k = 1 is a
    plain SwiGLU FFN;
  * brute force over all k-subsets on tiny shapes;
  * invariants: weights sum to 1, counts sum to T*k, capacity bookkeeping,
    unselected experts do not matter, token-permutation invariance;
  * load-balance statistics: importance against the routing weights at
    k = E, the logistic closed form and uniform cases; the penalties against
    transformers' Mixtral load-balancing loss and the torch calls (kl_div,
    std) the pages' snippets make;
  * hand-built golden fixtures under tests/golden/.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f64(a, dtype):
    """Exact fp64 view of generator output (bf16 bits or float32)."""
    return (mi.bf16_bits_to_f32(a) if dtype == "bf16" else a).astype(np.float64)


def small(T=37, H=48, I=40, E=6, k=2, dtype="f32", **kw):
    return mi.Workload("pin", T=T, H=H, I=I, E=E, k=k, dtype=dtype, **kw)


# ---------------------------------------------------------------- routing

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("E,k", [(8, 2), (32, 4), (16, 1)])
def test_route_matches_transformers_topk_softmax_router(dtype, E, k):
    """gpt-oss router in transformers: logits with bias, top-k, softmax over the k (fp64)."""
    from transformers import GptOssConfig
    from transformers.models.gpt_oss.modeling_gpt_oss import GptOssTopKRouter

    wl = small(T=50, H=40, E=E, k=k, dtype=dtype, zipf_s=1.1)
    inp = mi.make_inputs(wl)
    cfg = GptOssConfig(hidden_size=wl.H, num_local_experts=E, num_experts_per_tok=k)
    r = GptOssTopKRouter(cfg).double()
    with torch.no_grad():
        r.weight.copy_(torch.from_numpy(f64(inp["router_w"], dtype)))
        r.bias.copy_(torch.from_numpy(inp["router_b"].astype(np.float64)))
        logits_ref, w_ref, idx_ref = r(torch.from_numpy(f64(inp["x"], dtype)))
    logits, idx, w = oracle.route(inp["x"], inp["router_w"], inp["router_b"], k, dtype)
    np.testing.assert_allclose(logits, logits_ref.numpy(), rtol=0, atol=1e-12)
    assert np.array_equal(idx, idx_ref.numpy())
    np.testing.assert_allclose(w, w_ref.numpy(), rtol=0, atol=1e-14)


def test_route_logits_equal_float64_matmul_plus_bias():
    wl = small(T=64, H=96, E=16, k=3, dtype="bf16", zipf_s=1.1)
    inp = mi.make_inputs(wl)
    logits, _, _ = oracle.route(inp["x"], inp["router_w"], inp["router_b"], wl.k, wl.dtype)
    ref = f64(inp["x"], "bf16") @ f64(inp["router_w"], "bf16").T + inp["router_b"].astype(np.float64)
    np.testing.assert_allclose(logits, ref, rtol=0, atol=1e-12)


def test_route_brute_force_subsets():
    """The selected set maximises the sum of scores over all k-subsets; equal sums
    go to the lexicographically smallest sorted tuple (lower indices first)."""
    rng_wl = small(T=40, H=8, E=7, k=3, dtype="f32")
    inp = mi.make_inputs(rng_wl)
    # force some exact ties: a bias with repeated values and a zero-input token
    inp["x"][:5] = 0.0
    inp["router_b"] = np.array([0.5, 1.0, 1.0, -2.0, 1.0, 0.5, 0.0], np.float32)
    logits, idx, _ = oracle.route(inp["x"], inp["router_w"], inp["router_b"], 3, "f32")
    for t in range(rng_wl.T):
        best, best_key = None, None
        for sub in itertools.combinations(range(7), 3):
            key = (-math.fsum(logits[t, list(sub)]), sub)
            if best_key is None or key < best_key:
                best, best_key = sub, key
        # sum-maximal sets can differ only under ties; with ties the lower
        # indices win elementwise, which is the lexicographic minimum here
        assert tuple(sorted(idx[t])) == best, t
    # ordering within a token: score descending, then index ascending
    for t in range(rng_wl.T):
        keys = [(-logits[t, e], e) for e in idx[t]]
        assert keys == sorted(keys)


def test_route_ties_golden():
    g = json.load(open(os.path.join(GOLDEN, "route_ties.json")))
    for case in g["cases"]:
        b = np.array(case["bias"], np.float32)
        E, k, H = len(b), case["k"], 4
        x = np.zeros((3, H), np.float32)
        rw = mi.normal(0, 99, (E, H), 1.0, "f32")
        _, idx, w = oracle.route(x, rw, b, k, "f32")
        for t in range(3):
            assert idx[t].tolist() == case["topk_idx"]
            if case["topk_w"] is not None:
                np.testing.assert_allclose(w[t], case["topk_w"], rtol=0, atol=1e-7)


def test_two_way_softmax_is_logistic_and_k1_weight_is_one():
    wl = small(T=200, H=32, E=8, k=2)
    inp = mi.make_inputs(wl)
    logits, idx, w = oracle.route(inp["x"], inp["router_w"], None, 2, "f32")
    d = logits[np.arange(wl.T), idx[:, 0]] - logits[np.arange(wl.T), idx[:, 1]]
    np.testing.assert_allclose(w[:, 0], 1.0 / (1.0 + np.exp(-d)), rtol=0, atol=1e-15)
    _, _, w1 = oracle.route(inp["x"], inp["router_w"], None, 1, "f32")
    assert np.all(w1 == 1.0)


@pytest.mark.parametrize("E,k", [(8, 2), (128, 8), (256, 8)])
def test_weights_sum_to_one_and_follow_scores(E, k):
    wl = small(T=300, H=64, E=E, k=k, dtype="bf16", zipf_s=1.1)
    inp = mi.make_inputs(wl)
    logits, idx, w = oracle.route(inp["x"], inp["router_w"], inp["router_b"], k, "bf16")
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=1e-15)
    assert np.all(w > 0)
    assert np.all(np.diff(w, axis=1) <= 0)
    # softmax over all E, take top-k, renormalise == top-k then softmax over the k
    p = np.exp(logits - logits.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    pk = np.take_along_axis(p, idx, 1)
    np.testing.assert_allclose(pk / pk.sum(1, keepdims=True), w, rtol=0, atol=1e-15)
    # the selected probabilities are the k largest of the full softmax
    assert np.all(pk.min(1) >= np.sort(p, 1)[:, -k] - 1e-15)


def test_topk_margin_golden():
    g = json.load(open(os.path.join(GOLDEN, "topk_margin.json")))
    for case in g["cases"]:
        m = oracle.topk_margin(np.array([case["logits"]], np.float64), case["k"])
        want = np.inf if case["margin"] is None else case["margin"]
        assert m.tolist() == [want], case


@pytest.mark.parametrize("E,k", [(8, 2), (32, 4), (256, 8), (7, 3)])
def test_topk_margin_is_the_smallest_gap_across_the_selection(E, k):
    """Brute force: the margin equals min over selected e and unselected e' of
    l_e - l_e', with the selection taken from the C oracle's routing."""
    wl = small(T=80, H=24, E=E, k=k, dtype="bf16", zipf_s=1.1)
    inp = mi.make_inputs(wl)
    logits, idx, _ = oracle.route(inp["x"], inp["router_w"], inp["router_b"], k, "bf16")
    m = oracle.topk_margin(logits, k)
    for t in range(wl.T):
        sel = set(idx[t].tolist())
        gaps = [logits[t, a] - logits[t, b] for a in sel for b in range(E) if b not in sel]
        assert m[t] == min(gaps), t
    # a zero-input token with a repeated bias: an exact tie across the boundary
    x0 = np.zeros((1, 8), np.float32)
    b = np.array([2.0, 1.0, 1.0, 0.0], np.float32)
    l0, _, _ = oracle.route(x0, mi.normal(0, 99, (4, 8), 1.0, "f32"), b, 2, "f32")
    assert oracle.topk_margin(l0, 2).tolist() == [0.0]
    assert oracle.topk_margin(l0, 4).tolist() == [np.inf]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_weights_for_equals_route_weights_and_transformers_router(dtype):
    """weights_for on the oracle's own selection reproduces the C oracle's
    weights and transformers' GptOssTopKRouter weights (fp64), in any order of
    the selection; k = 1 gives exactly 1."""
    from transformers import GptOssConfig
    from transformers.models.gpt_oss.modeling_gpt_oss import GptOssTopKRouter

    wl = small(T=60, H=40, E=16, k=4, dtype=dtype, zipf_s=1.1)
    inp = mi.make_inputs(wl)
    logits, idx, w = oracle.route(inp["x"], inp["router_w"], inp["router_b"], wl.k, dtype)
    got = oracle.weights_for(logits, idx)
    np.testing.assert_allclose(got, w, rtol=0, atol=1e-14)
    cfg = GptOssConfig(hidden_size=wl.H, num_local_experts=wl.E, num_experts_per_tok=wl.k)
    r = GptOssTopKRouter(cfg).double()
    with torch.no_grad():
        r.weight.copy_(torch.from_numpy(f64(inp["router_w"], dtype)))
        r.bias.copy_(torch.from_numpy(inp["router_b"].astype(np.float64)))
        _, w_ref, idx_ref = r(torch.from_numpy(f64(inp["x"], dtype)))
    np.testing.assert_allclose(oracle.weights_for(logits, idx_ref.numpy()), w_ref.numpy(), rtol=0, atol=1e-14)
    rev = idx[:, ::-1]
    np.testing.assert_allclose(oracle.weights_for(logits, rev), got[:, ::-1], rtol=0, atol=1e-15)
    assert np.all(oracle.weights_for(logits, idx[:, :1]) == 1.0)


def test_capacity_golden():
    g = json.load(open(os.path.join(GOLDEN, "capacity_formula.json")))
    for c in g["cases"]:
        assert oracle.capacity(c["cf"], c["T"], c["k"], c["E"]) == c["C"], c
    assert oracle.capacity(mi.QWEN3.capacity_factor, mi.QWEN3.T, mi.QWEN3.k, mi.QWEN3.E) == 2560
    assert oracle.capacity(mi.MIXTRAL.capacity_factor, mi.MIXTRAL.T, mi.MIXTRAL.k, mi.MIXTRAL.E) == 0


# ------------------------------------------------- load-balance statistics

def test_importance_with_top_k_equal_E_is_the_sum_of_routing_weights():
    """With k = E the routing weights are the softmax over all E scores, so
    their per-expert sum over tokens is the importance (and it sums to T)."""
    wl = small(T=90, H=40, E=16, k=16, dtype="bf16", zipf_s=1.1)
    inp = mi.make_inputs(wl)
    logits, idx, w = oracle.route(inp["x"], inp["router_w"], inp["router_b"], wl.k, wl.dtype)
    from_route = np.zeros(wl.E)
    np.add.at(from_route, idx.ravel(), w.ravel())
    imp = oracle.importance(logits)
    np.testing.assert_allclose(imp, from_route, rtol=1e-13, atol=0)
    assert abs(imp.sum() - wl.T) <= 1e-12 * wl.T


def test_importance_of_two_experts_is_a_sum_of_logistics():
    wl = small(T=120, H=32, E=2, k=1)
    inp = mi.make_inputs(wl)
    logits, _, _ = oracle.route(inp["x"], inp["router_w"], None, 1, "f32")
    imp = oracle.importance(logits)
    ref0 = np.sum(1.0 / (1.0 + np.exp(logits[:, 1] - logits[:, 0])))
    assert abs(imp[0] - ref0) <= 1e-12 * wl.T
    assert abs(imp[1] - (wl.T - ref0)) <= 1e-12 * wl.T


def test_importance_of_identical_router_rows_is_uniform():
    wl = small(T=33, H=24, E=8, k=2)
    inp = mi.make_inputs(wl)
    rw = np.repeat(inp["router_w"][:1], wl.E, axis=0)
    logits, _, _ = oracle.route(inp["x"], rw, None, wl.k, "f32")
    assert np.array_equal(oracle.importance(logits), np.full(wl.E, wl.T / wl.E))


def test_importance_follows_a_permutation_of_the_experts():
    wl = small(T=64, H=32, E=12, k=3, dtype="bf16", zipf_s=1.1)
    inp = mi.make_inputs(wl)
    perm = np.random.default_rng(3).permutation(wl.E)
    l1, _, _ = oracle.route(inp["x"], inp["router_w"], inp["router_b"], wl.k, wl.dtype)
    l2, _, _ = oracle.route(inp["x"], inp["router_w"][perm], inp["router_b"][perm], wl.k, wl.dtype)
    np.testing.assert_allclose(oracle.importance(l2), oracle.importance(l1)[perm], rtol=1e-14, atol=0)


def test_importance_and_penalties_golden():
    g = json.load(open(os.path.join(GOLDEN, "importance_bias_only.json")))
    for case in g["cases"]:
        b = np.array(case["bias"], np.float32)
        E, T, k = len(b), case["T"], case["k"]
        x = np.zeros((T, 8), np.float32)
        rw = mi.normal(0, 99, (E, 8), 1.0, "f32")
        logits, idx, _ = oracle.route(x, rw, b, k, "f32")
        imp = oracle.importance(logits)
        np.testing.assert_allclose(imp, case["importance"], rtol=1e-7, atol=0)
        if case["load"] is not None:
            load = oracle.permute(idx, E)["counts"]
            assert load.tolist() == case["load"]
            got = oracle.balance_losses(imp, load, T)
            for key in ("kl", "std", "switch"):
                assert abs(got[key] - case[key]) <= 1e-6 * abs(case[key]), key


def test_switch_loss_matches_transformers_mixtral_load_balancing():
    from transformers.models.mixtral.modeling_mixtral import load_balancing_loss_func
    wl = small(T=200, H=48, E=8, k=2, dtype="bf16", zipf_s=1.1)
    inp = mi.make_inputs(wl)
    logits, idx, _ = oracle.route(inp["x"], inp["router_w"], inp["router_b"], wl.k, wl.dtype)
    counts = oracle.permute(idx, wl.E)["counts"]
    got = oracle.balance_losses(oracle.importance(logits), counts, wl.T)["switch"]
    ref = load_balancing_loss_func((torch.from_numpy(logits),), wl.E, wl.k).item()
    assert abs(got - ref) <= 1e-9 * abs(ref)


@pytest.mark.parametrize("case", ["uniform", "collapsed", "random"])
def test_kl_and_std_losses_match_the_torch_calls_of_the_pages(case):
    """KL: torch.nn.functional.kl_div(log(q + 1e-8), 1/E, reduction="batchmean")
    on the mean gate probability q; std: torch.std (unbiased) of importance and
    load, the calls the pages' snippets make."""
    E, T = 8, 100
    if case == "uniform":
        imp, load = np.full(E, T / E), np.full(E, 25.0)
    elif case == "collapsed":
        imp, load = np.eye(E)[0] * T, np.eye(E)[0] * 2 * T
    else:
        rng = np.random.default_rng(7)
        imp = rng.dirichlet(np.ones(E)) * T
        load = rng.integers(0, 2 * T, E).astype(np.float64)
    got = oracle.balance_losses(imp, load, T)
    q = torch.from_numpy(imp / T)
    kl = torch.nn.functional.kl_div(torch.log(q + 1e-8), torch.full((E,), 1.0 / E, dtype=torch.float64),
                                    reduction="batchmean").item()
    std = (torch.std(torch.from_numpy(imp)) + torch.std(torch.from_numpy(load))).item()
    assert abs(got["kl"] - kl) <= 1e-12 * max(1.0, abs(kl))
    assert abs(got["std"] - std) <= 1e-12 * max(1.0, abs(std))
    if case == "uniform":
        assert got["std"] == 0.0 and abs(got["kl"] + math.log1p(E * 1e-8) / E) < 1e-15
        assert abs(got["switch"] - 2.0) < 1e-12  # E * sum (2T/E / T)(1/E) = k with k = 2


# ---------------------------------------------------------------- grouping

@pytest.mark.parametrize("name", ["capacity_toy.json", "capacity_toy_k2.json"])
def test_permute_golden(name):
    g = json.load(open(os.path.join(GOLDEN, name)))
    r = oracle.permute(np.array(g["topk_idx"], np.int32), g["E"], g["capacity"])
    for key in ("counts", "dropped", "offsets", "perm_rows", "row_of"):
        assert r[key].tolist() == g[key], key


@pytest.mark.parametrize("cf", [0.0, 1.0, 1.25, 2.0])
def test_permute_invariants(cf):
    wl = small(T=3000, H=16, E=128, k=8, dtype="f32", zipf_s=1.1, capacity_factor=cf)
    inp = mi.make_inputs(wl)
    _, idx, _ = oracle.route(inp["x"], inp["router_w"], inp["router_b"], wl.k, "f32")
    C = oracle.capacity(wl.capacity_factor, wl.T, wl.k, wl.E)
    r = oracle.permute(idx, wl.E, C)
    counts, dropped, off = r["counts"], r["dropped"], r["offsets"]
    assert counts.sum() == wl.T * wl.k
    assert np.array_equal(counts, np.bincount(idx.ravel(), minlength=wl.E))
    kept = np.minimum(counts, C) if C > 0 else counts
    assert np.array_equal(np.diff(off), kept)
    assert np.array_equal(dropped, counts - kept)
    assert kept.sum() + dropped.sum() == wl.T * wl.k
    R = off[-1]
    pr, ro = r["perm_rows"], r["row_of"].ravel()
    assert np.all(pr[R:] == -1) and np.all(pr[:R] >= 0)
    assert np.array_equal(ro[pr[:R]], np.arange(R))          # bijection rows <-> kept slots
    assert (ro >= 0).sum() == R
    for e in range(wl.E):
        rows = pr[off[e]:off[e + 1]]
        assert np.all(idx.ravel()[rows] == e)
        tok = rows // wl.k
        assert np.all(np.diff(tok) > 0)                      # ascending token order
        if C > 0 and counts[e] > C:                          # the earliest C tokens are kept
            all_tok = np.nonzero((idx == e).any(1))[0]
            assert np.array_equal(tok, all_tok[:C])


# ---------------------------------------------------------------- experts

def _mixtral_experts(inp, dtype, E, H, I):
    from transformers import MixtralConfig
    from transformers.models.mixtral.modeling_mixtral import MixtralExperts

    cfg = MixtralConfig(hidden_size=H, intermediate_size=I, num_local_experts=E, hidden_act="silu")
    m = MixtralExperts(cfg).double()
    with torch.no_grad():
        gu = np.concatenate([f64(inp["w_gate"], dtype), f64(inp["w_up"], dtype)], axis=1)
        m.gate_up_proj.copy_(torch.from_numpy(gu))
        m.down_proj.copy_(torch.from_numpy(f64(inp["w_down"], dtype)))
    return m


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_experts_match_transformers_mixtral_experts(dtype):
    """Weighted sum of the selected SwiGLU experts == transformers' eager packed experts."""
    wl = small(T=45, H=40, I=24, E=6, k=2, dtype=dtype)
    inp = mi.make_inputs(wl)
    _, idx, w = oracle.route(inp["x"], inp["router_w"], None, wl.k, dtype)
    y = oracle.moe_tokens(inp["x"], inp["w_gate"], inp["w_up"], inp["w_down"], idx, w, dtype)
    m = _mixtral_experts(inp, dtype, wl.E, wl.H, wl.I)
    with torch.no_grad():
        ref = m(torch.from_numpy(f64(inp["x"], dtype)), torch.from_numpy(idx.astype(np.int64)),
                torch.from_numpy(w)).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-13)


def test_full_layer_matches_transformers_mixtral_block():
    """Mixtral's block: softmax over all E (float32), top-k, renormalise."""
    from transformers import MixtralConfig
    from transformers.models.mixtral.modeling_mixtral import MixtralSparseMoeBlock

    wl = small(T=64, H=32, I=48, E=8, k=2, dtype="f32")
    inp = mi.make_inputs(wl)
    cfg = MixtralConfig(hidden_size=wl.H, intermediate_size=wl.I, num_local_experts=wl.E,
                        num_experts_per_tok=wl.k, hidden_act="silu")
    blk = MixtralSparseMoeBlock(cfg).double().eval()
    with torch.no_grad():
        blk.gate.weight.copy_(torch.from_numpy(f64(inp["router_w"], "f32")))
        gu = np.concatenate([f64(inp["w_gate"], "f32"), f64(inp["w_up"], "f32")], axis=1)
        blk.experts.gate_up_proj.copy_(torch.from_numpy(gu))
        blk.experts.down_proj.copy_(torch.from_numpy(f64(inp["w_down"], "f32")))
        ref = blk(torch.from_numpy(f64(inp["x"], "f32"))[None])[0].numpy()
    out = oracle.forward(wl, inp)
    assert np.all(out["margin"] > 1e-5)
    np.testing.assert_allclose(out["y"], ref, rtol=1e-5, atol=1e-6)


def test_single_expert_is_dense_swiglu_ffn():
    """E = k = 1: weight exactly 1 and y = W_d (silu(W_g x) * W_u x) via torch float64."""
    wl = small(T=20, H=24, I=56, E=1, k=1, dtype="bf16")
    inp = mi.make_inputs(wl)
    out = oracle.forward(wl, inp)
    assert np.all(out["topk_w"] == 1.0) and np.all(out["topk_idx"] == 0)
    x = torch.from_numpy(f64(inp["x"], "bf16"))
    g = torch.from_numpy(f64(inp["w_gate"], "bf16")[0])
    u = torch.from_numpy(f64(inp["w_up"], "bf16")[0])
    d = torch.from_numpy(f64(inp["w_down"], "bf16")[0])
    ref = torch.nn.functional.linear(torch.nn.functional.silu(x @ g.T) * (x @ u.T), d).numpy()
    np.testing.assert_allclose(out["y"], ref, rtol=1e-12, atol=1e-13)


def test_swiglu_closed_form_scalar():
    """H = I = 1, unit weights: y = silu(x) * x = x^2 / (1 + e^-x)."""
    x = np.array([[2.0], [-3.0], [0.0], [0.5]], np.float32)
    one = np.ones((1, 1, 1), np.float32)
    y = oracle.moe_tokens(x, one, one, one, np.zeros((4, 1), np.int32), np.ones((4, 1)), "f32")
    for t, v in enumerate([2.0, -3.0, 0.0, 0.5]):
        assert y[t, 0] == pytest.approx(v * v / (1.0 + math.exp(-v)), rel=1e-15, abs=1e-300)


def test_shared_expert_is_added_with_weight_one():
    wl = small(T=30, H=40, I=24, E=6, k=2, dtype="bf16", I_shared=32)
    inp = mi.make_inputs(wl)
    out = oracle.forward(wl, inp)
    routed = oracle.moe_tokens(inp["x"], inp["w_gate"], inp["w_up"], inp["w_down"], out["topk_idx"],
                               out["topk_w"], "bf16")
    sh = {"w_gate": inp["ws_gate"][None], "w_up": inp["ws_up"][None], "w_down": inp["ws_down"][None]}
    m = _mixtral_experts(sh, "bf16", 1, wl.H, wl.I_shared)
    with torch.no_grad():
        ref = m(torch.from_numpy(f64(inp["x"], "bf16")), torch.zeros((wl.T, 1), dtype=torch.int64),
                torch.ones((wl.T, 1), dtype=torch.float64)).numpy()
    np.testing.assert_allclose(out["y"] - routed, ref, rtol=1e-11, atol=1e-12)


def test_top_k_equal_E_is_dense_softmax_mixture():
    """With k = E every expert is chosen: y = sum_e softmax(l)_e FFN_e(x)."""
    wl = small(T=25, H=32, I=20, E=5, k=5, dtype="f32")
    inp = mi.make_inputs(wl)
    out = oracle.forward(wl, inp)
    l = f64(inp["x"], "f32") @ f64(inp["router_w"], "f32").T
    p = torch.softmax(torch.from_numpy(l), dim=1)
    m = _mixtral_experts(inp, "f32", wl.E, wl.H, wl.I)
    dense = np.zeros((wl.T, wl.H))
    x = torch.from_numpy(f64(inp["x"], "f32"))
    with torch.no_grad():
        for e in range(wl.E):   # every expert on every token, mixed by the full softmax
            ye = m(x, torch.full((wl.T, 1), e, dtype=torch.int64), torch.ones((wl.T, 1), dtype=torch.float64))
            dense += p[:, e:e + 1].numpy() * ye.numpy()
    np.testing.assert_allclose(out["y"], dense, rtol=1e-12, atol=1e-13)


def test_unselected_experts_do_not_change_output():
    wl = small(T=6, H=32, I=16, E=16, k=2, dtype="bf16")
    inp = mi.make_inputs(wl)
    out = oracle.forward(wl, inp)
    unused = sorted(set(range(wl.E)) - set(out["topk_idx"].ravel().tolist()))
    assert unused
    inp2 = dict(inp)
    for key in ("w_gate", "w_up", "w_down"):
        inp2[key] = inp[key].copy()
        inp2[key][unused] = mi.normal(7, 77, inp[key][unused].shape, 3.0, "bf16")
    out2 = oracle.forward(wl, inp2)
    assert np.array_equal(out["y"], out2["y"])


def test_token_permutation_invariance():
    wl = small(T=40, H=32, I=16, E=8, k=3, dtype="bf16", I_shared=8)
    inp = mi.make_inputs(wl)
    out = oracle.forward(wl, inp)
    pi = mi.permutation(3, 1, wl.T)
    inp2 = dict(inp, x=inp["x"][pi])
    out2 = oracle.forward(wl, inp2)
    assert np.array_equal(out2["y"], out["y"][pi])
    assert np.array_equal(out2["topk_idx"], out["topk_idx"][pi])


def test_dropped_pairs_contribute_nothing():
    wl = small(T=400, H=32, I=16, E=8, k=2, dtype="f32", capacity_factor=0.5)
    inp = mi.make_inputs(wl)
    out = oracle.forward(wl, inp)
    ro = out["row_of"]
    assert (ro < 0).any()
    w_kept = np.where(ro >= 0, out["topk_w"], 0.0)
    y_ref = oracle.moe_tokens(inp["x"], inp["w_gate"], inp["w_up"], inp["w_down"], out["topk_idx"],
                              w_kept, "f32")
    np.testing.assert_allclose(out["y"], y_ref, rtol=1e-13, atol=1e-14)
    all_dropped = np.all(ro < 0, axis=1)
    assert np.all(out["y"][all_dropped] == 0.0)


def test_sampled_tokens_equal_full_evaluation():
    wl = small(T=50, H=32, I=16, E=8, k=2, dtype="bf16")
    inp = mi.make_inputs(wl)
    full = oracle.forward(wl, inp)
    tok = mi.sample_tokens(5, wl.T, 9)
    part = oracle.forward(wl, inp, tokens=tok)
    assert np.array_equal(part["y"], full["y"][tok])


# ------------------------------------------------------------- mxfp4 weights
# The FP4 E2M1 value table of the OCP Microscaling v1.0 specification
# (magnitudes of codes 0..7; codes 8..15 are their negatives).
E2M1_SPEC = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_codes_match_the_specification_table():
    spec = E2M1_SPEC + [-v for v in E2M1_SPEC]
    assert [oracle.e2m1_value(c) for c in range(16)] == spec
    # all 16 codes through the block path, scale byte 127 = 2^0
    codes = np.arange(32) % 16
    blocks = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)[None, :]
    got = oracle.mxfp4_dequantize(blocks, np.array([127], np.uint8))
    assert got.tolist() == [spec[c] for c in codes]
    assert math.copysign(1.0, got[8]) == -1.0  # code 8 is -0


def test_mxfp4_scale_bytes_are_powers_of_two():
    blocks = np.full((255, 1, 16), 0x22, np.uint8)  # every element code 2 = 1.0
    scales = np.arange(255, dtype=np.uint8)[:, None]
    got = oracle.mxfp4_dequantize(blocks, scales)
    for s in range(255):
        assert np.all(got[s] == math.ldexp(1.0, s - 127)), s
    nan = oracle.mxfp4_dequantize(blocks[:1], np.array([[255]], np.uint8))
    assert np.all(np.isnan(nan))


def test_mxfp4_nan_scale_propagates_to_the_tokens_that_read_it():
    """A scale byte of 255 (the specification's NaN) in one block of one
    expert's gate row: every token routed to that expert gets NaN outputs,
    the other tokens are unchanged."""
    wl = small(T=10, H=64, I=32, E=3, k=1, dtype="bf16")
    inp = mi.make_inputs(wl, router_only=True)
    mx = mi.make_mxfp4_experts(wl)
    idx = (np.arange(wl.T) % wl.E).astype(np.int32)[:, None]
    w = np.ones((wl.T, 1))
    y0 = oracle.moe_tokens_mxfp4(inp["x"], mx, idx, w, "bf16")
    blocks, scales = mx["w_gate"]
    scales = scales.copy()
    scales[1, 5, 1] = 255  # expert 1, gate row 5, second block
    mx2 = dict(mx, w_gate=(blocks, scales))
    y1 = oracle.moe_tokens_mxfp4(inp["x"], mx2, idx, w, "bf16")
    hit = idx[:, 0] == 1
    assert np.all(np.isnan(y1[hit]))
    assert np.array_equal(y1[~hit], y0[~hit])


def test_mxfp4_nibble_order_and_per_block_scales():
    """Hand-built row of two blocks: bytes 0x21, 0xF0 in block 0 (scale 2^0)
    and 0x76 in block 1 (scale 2^1): elements 0.5, 1, 0, -6, ... and 8, 12."""
    blocks = np.zeros((2, 16), np.uint8)
    blocks[0, 0], blocks[0, 1], blocks[1, 0] = 0x21, 0xF0, 0x76
    got = oracle.mxfp4_dequantize(blocks, np.array([127, 128], np.uint8))
    assert got.shape == (64,)
    assert got[:4].tolist() == [0.5, 1.0, 0.0, -6.0] and np.all(got[4:32] == 0)
    assert got[32:34].tolist() == [8.0, 12.0] and np.all(got[34:] == 0)


def test_mxfp4_single_expert_is_dense_swiglu_ffn():
    """E = k = 1 with mxfp4 weights: y = W_d (silu(W_g x) * W_u x) on the
    dequantized weights, via torch float64."""
    wl = small(T=12, H=64, I=96, E=1, k=1, dtype="bf16")
    inp = mi.make_inputs(wl, router_only=True)
    mx = mi.make_mxfp4_experts(wl)
    idx = np.zeros((wl.T, 1), np.int32)
    y = oracle.moe_tokens_mxfp4(inp["x"], mx, idx, np.ones((wl.T, 1)), "bf16")
    x = torch.from_numpy(f64(inp["x"], "bf16"))
    g, u, d = (torch.from_numpy(oracle.mxfp4_dequantize(*mx[n])[0]) for n in ("w_gate", "w_up", "w_down"))
    ref = torch.nn.functional.linear(torch.nn.functional.silu(x @ g.T) * (x @ u.T), d).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-13 * np.abs(ref).max())


# ---------------------------------------------------------------- backward

def _torch_layer_grads(inp, dtype, idx, row_of, dy):
    """The layer in torch float64 with the selection held fixed (top-k and the
    capacity cut carry no gradient), differentiated by autograd."""
    def t64(a):
        return torch.from_numpy(f64(a, dtype)).requires_grad_(True) if a is not None else None

    x, rw, wg, wu, wd = (t64(inp[n]) for n in ("x", "router_w", "w_gate", "w_up", "w_down"))
    rb = torch.from_numpy(inp["router_b"].astype(np.float64)).requires_grad_(True) \
        if inp["router_b"] is not None else None
    sg, su, sd = (t64(inp[n]) for n in ("ws_gate", "ws_up", "ws_down"))
    T, k = idx.shape
    logits = x @ rw.T + (rb if rb is not None else 0.0)
    w = torch.softmax(torch.gather(logits, 1, torch.from_numpy(idx.astype(np.int64))), dim=1)
    rows = []
    for t in range(T):
        yt = torch.zeros(x.shape[1], dtype=torch.float64)
        for j in range(k):
            if row_of[t, j] < 0:
                continue
            e = int(idx[t, j])
            a = torch.nn.functional.silu(wg[e] @ x[t]) * (wu[e] @ x[t])
            yt = yt + w[t, j] * (wd[e] @ a)
        if sg is not None:
            yt = yt + sd @ (torch.nn.functional.silu(sg @ x[t]) * (su @ x[t]))
        rows.append(yt)
    y = torch.stack(rows)
    (y * torch.from_numpy(dy)).sum().backward()
    out = dict(dx=x.grad, d_router_w=rw.grad, d_w_gate=wg.grad, d_w_up=wu.grad, d_w_down=wd.grad)
    out["d_router_b"] = rb.grad if rb is not None else None
    if sg is not None:
        out.update(d_ws_gate=sg.grad, d_ws_up=su.grad, d_ws_down=sd.grad)
    return {kk: (v.numpy() if v is not None else None) for kk, v in out.items()}


@pytest.mark.parametrize("case", [
    dict(T=24, H=32, I=24, E=6, k=2, dtype="bf16", zipf_s=1.1, I_shared=16, capacity_factor=0.6),
    dict(T=20, H=24, I=16, E=8, k=3, dtype="f32"),
    dict(T=16, H=16, I=8, E=4, k=4, dtype="f32", zipf_s=1.1),
], ids=["bf16_bias_shared_drops", "f32_k3", "f32_k_eq_E"])
def test_backward_matches_torch_autograd(case):
    """Every gradient of the layer against autograd through a float64 torch
    restatement of the forward, the selection and capacity cut held fixed."""
    wl = small(**case)
    inp = mi.make_inputs(wl)
    if inp["router_b"] is None:
        inp["router_b"] = np.zeros(wl.E, np.float32)
    _, idx, w = oracle.route(inp["x"], inp["router_w"], inp["router_b"], wl.k, wl.dtype)
    row_of = oracle.permute(idx, wl.E, oracle.capacity(wl.capacity_factor, wl.T, wl.k, wl.E))["row_of"]
    if wl.capacity_factor > 0:
        assert (row_of < 0).any()
    dy = mi.normal(3, 77, (wl.T, wl.H), 1.0, "f32").astype(np.float64)
    got = oracle.moe_backward(inp["x"], inp["router_w"], inp["w_gate"], inp["w_up"], inp["w_down"], idx, w, dy,
                              wl.dtype, row_of=row_of, ws_gate=inp["ws_gate"], ws_up=inp["ws_up"],
                              ws_down=inp["ws_down"])
    ref = _torch_layer_grads(inp, wl.dtype, idx, row_of, dy)
    for name, r in ref.items():
        scale = max(np.abs(r).max(), 1e-300)
        assert np.max(np.abs(got[name] - r)) <= 1e-11 * scale, name


def test_backward_top1_routes_no_gradient_to_the_router():
    """k = 1: the softmax over one score is 1 whatever the score, so the
    router gets exactly zero gradient; unselected experts get exactly zero."""
    wl = small(T=30, H=24, I=16, E=8, k=1, dtype="f32")
    inp = mi.make_inputs(wl)
    _, idx, w = oracle.route(inp["x"], inp["router_w"], None, 1, "f32")
    dy = mi.normal(4, 78, (wl.T, wl.H), 1.0, "f32").astype(np.float64)
    got = oracle.moe_backward(inp["x"], inp["router_w"], inp["w_gate"], inp["w_up"], inp["w_down"], idx, w, dy,
                              "f32")
    assert np.all(got["d_router_w"] == 0.0) and np.all(got["d_router_b"] == 0.0)
    unused = sorted(set(range(wl.E)) - set(idx.ravel().tolist()))
    for e in unused:
        assert np.all(got["d_w_gate"][e] == 0) and np.all(got["d_w_down"][e] == 0)
    # the router's part of dx is zero too: dx equals the experts' part alone
    assert np.all(np.isfinite(got["dx"]))


def test_backward_dropped_pairs_carry_only_the_router_gradient():
    """A pair dropped by the capacity cut adds nothing to y, so its expert
    gets no gradient from it; its weight still enters the softmax."""
    wl = small(T=40, H=16, I=8, E=4, k=2, dtype="f32", capacity_factor=0.3)
    inp = mi.make_inputs(wl)
    _, idx, w = oracle.route(inp["x"], inp["router_w"], None, 2, "f32")
    row_of = oracle.permute(idx, wl.E, oracle.capacity(0.3, wl.T, 2, wl.E))["row_of"]
    dy = mi.normal(5, 79, (wl.T, wl.H), 1.0, "f32").astype(np.float64)
    kept_only = oracle.moe_backward(inp["x"], inp["router_w"], inp["w_gate"], inp["w_up"], inp["w_down"], idx, w,
                                    dy, "f32", row_of=row_of)
    # the same layer evaluated on just the kept pairs' tokens gives the
    # expert weight gradients: a token whose pairs are all dropped adds none
    all_dropped = np.all(row_of < 0, axis=1)
    assert all_dropped.any()
    # a token with every pair dropped has dw = 0, hence dl = 0: no gradient at all
    assert np.all(kept_only["dx"][all_dropped] == 0.0)
    dy2 = dy.copy()
    dy2[all_dropped] = 0.0
    other = oracle.moe_backward(inp["x"], inp["router_w"], inp["w_gate"], inp["w_up"], inp["w_down"], idx, w,
                                dy2, "f32", row_of=row_of)
    for name in ("d_w_gate", "d_w_up", "d_w_down"):
        np.testing.assert_allclose(other[name], kept_only[name], rtol=0, atol=1e-13)
