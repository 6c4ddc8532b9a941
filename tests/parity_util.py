"""Shared helpers of the GPU parity tests: device copies of the seeded inputs,
the routing comparison with the near-tie exemption, and the output metric.

Rules (the layer's stated parity contract):
  * expert sets, their order within a token (score descending, ties to the
    lower index) and per-expert counts / offsets / dropped counts match the
    oracle bit-exactly, except for tokens whose k-th/(k+1)-th oracle logit
    margin is in (0, 1e-5); for those any selection whose every score is
    within 1e-5 of the k-th largest is accepted, and the oracle is
    re-evaluated on the GPU's selection (weights, grouping, outputs); two
    selected scores within (0, 1e-5) may come in either order; exact ties
    are never exempt;
  * outputs: max over tokens of ||y_t - yhat_t||_inf / ||yhat_t||_inf is at
    most 2e-2 for bf16 and 1e-4 for float32; rows whose oracle output is
    exactly 0 (every pair dropped) must be exactly 0.
"""
import numpy as np
import torch

import moe_inputs as mi
import oracle

TIE_MARGIN = 1e-5
TOL = {"bf16": 2e-2, "f32": 1e-4}


def cap_of(wl) -> int:
    """The oracle's per-expert capacity of workload wl (0 = unlimited)."""
    return oracle.capacity(wl.capacity_factor, wl.T, wl.k, wl.E)


def dev(a, dtype):
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def to_device(inp: dict, dtype: str) -> dict:
    return {k: dev(v, dtype) for k, v in inp.items()}


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def adjacent_gaps(logits, idx):
    """Score gaps between consecutive selected experts of each token, in the
    given order: [T, k-1] (positive when the order is score-descending)."""
    lg = np.take_along_axis(logits, idx.astype(np.int64), 1)
    return lg[:, :-1] - lg[:, 1:]


def check_selection(logits, idx_o, margin, idx_g, k):
    """Returns the boolean exempt mask; asserts the selection and order rules.

    Selection: the expert set equals the oracle's, except for tokens whose
    k-th/(k+1)-th margin is in (0, 1e-5) (exempt: any selection whose every
    score is within 1e-5 of the k-th is accepted).  Order: the selected
    experts follow the exact order (score descending, ties to the lower
    index), so the ordered rows equal the oracle's, except where two selected
    scores are within (0, 1e-5) of each other, where either order is
    accepted.  Exact ties (gap 0) are never exempt: the lower index wins."""
    T = idx_o.shape[0]
    assert idx_g.shape == idx_o.shape
    exempt = (margin < TIE_MARGIN) & (margin > 0)
    so, sg = np.sort(idx_o, 1), np.sort(idx_g, 1)
    bad = np.nonzero(~exempt & np.any(so != sg, axis=1))[0]
    assert bad.size == 0, f"{bad.size} non-exempt tokens differ, first {bad[:5]}: " \
        f"oracle {idx_o[bad[:1]]} gpu {idx_g[bad[:1]]} margin {margin[bad[:1]]}"
    for t in np.nonzero(exempt)[0]:
        kth = np.sort(logits[t])[::-1][k - 1]
        assert len(set(idx_g[t].tolist())) == k
        assert np.all(logits[t, idx_g[t]] >= kth - TIE_MARGIN), t
    if k > 1:
        gaps = adjacent_gaps(logits, idx_o)
        near = np.any((gaps < TIE_MARGIN) & (gaps > 0), axis=1)
        strict = ~exempt & ~near
        wrong = np.nonzero(strict & np.any(idx_g != idx_o, axis=1))[0]
        assert wrong.size == 0, f"{wrong.size} tokens out of order, first {wrong[:5]}: " \
            f"oracle {idx_o[wrong[:1]]} gpu {idx_g[wrong[:1]]}"
        # elsewhere the order still follows the scores up to the exemption
        assert np.all(adjacent_gaps(logits, idx_g) >= -TIE_MARGIN)
    return exempt


def rowwise_rel_err(y, yhat):
    """max_t ||y_t - yhat_t||_inf / ||yhat_t||_inf over rows with yhat_t != 0;
    rows with yhat_t == 0 must be exactly zero (returns inf otherwise)."""
    den = np.abs(yhat).max(1)
    num = np.abs(y - yhat).max(1)
    zero = den == 0
    if np.any(num[zero] != 0):
        return float("inf")
    if np.all(zero):
        return 0.0
    return float(np.max(num[~zero] / den[~zero]))


def oracle_given_selection(wl, inp, logits, sel, tokens):
    """The oracle's layer output for `tokens`, with the routing selection `sel`
    (all T tokens) taken as given: weights, grouping and FFN from the oracle."""
    w = oracle.weights_for(logits, sel)
    perm = oracle.permute(sel, wl.E, cap_of(wl))
    y = oracle.moe_tokens(inp["x"], inp["w_gate"], inp["w_up"], inp["w_down"], sel, w, wl.dtype,
                          row_of=perm["row_of"], ws_gate=inp["ws_gate"], ws_up=inp["ws_up"],
                          ws_down=inp["ws_down"], tokens=tokens)
    return y, w, perm
