"""CPU oracle of the routed MoE FFN forward pass (fp64, plain C + OpenMP).

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import this
package.  It shares no code with the CUDA path (``sparse_mixture_experts_19_b200``);
both read their inputs from the seeded generator in ``moe_inputs``.

What it computes, per token (see ``moe_oracle.c`` for the sources):
score -> top-k (ties to the lower expert index) -> softmax over the k selected
scores -> capacity drop in token order -> weighted sum of the selected SwiGLU
experts (+ the always-on shared expert).  Router statistics for the
load-balance penalties: per-expert importance (sum over tokens of the softmax
over all E scores) and the penalties built from it and the top-k counts.
Expert weights in the MXFP4 microscaling format: dequantization from the
format's definition and the layer on those weights.  The backward pass:
every gradient of the layer by the chain rule through those steps.

Parity pins of every function here live in ``tests/test_oracle.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

DTYPE_CODE = {"f32": 0, "bf16": 1}


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so (gcc -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        _lib.oracle_route.argtypes = [i64, i32, i32, i32, i32, P, P, P, P, P, P]
        _lib.oracle_permute.argtypes = [i64, i32, i32, i64, P, P, P, P, P, P]
        _lib.oracle_moe_tokens.argtypes = [i64, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P,
                                           P, P, P, i64, P, P]
        _lib.oracle_moe_backward.argtypes = [i64, i32, i32, i32, i32, i32, i32] + [P] * 21
        for f in (_lib.oracle_route, _lib.oracle_permute, _lib.oracle_moe_tokens, _lib.oracle_moe_backward):
            f.restype = ctypes.c_int
        _lib.oracle_threads.argtypes = []
        _lib.oracle_threads.restype = ctypes.c_int
    return _lib


def threads() -> int:
    """OpenMP threads the oracle runs on."""
    return int(_L().oracle_threads())


def _ptr(a):
    return None if a is None else a.ctypes.data


def _c(a, dt=None):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=dt) if dt is not None else np.ascontiguousarray(a)


def route(x, router_w, router_b, k: int, dtype: str):
    """fp64 logits [T,E], topk_idx int32 [T,k], topk_w fp64 [T,k]."""
    x, router_w = _c(x), _c(router_w)
    router_b = _c(router_b, np.float32)
    T, H = x.shape
    E = router_w.shape[0]
    logits = np.empty((T, E), np.float64)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    rc = _L().oracle_route(T, H, E, k, DTYPE_CODE[dtype], _ptr(x), _ptr(router_w), _ptr(router_b),
                           _ptr(logits), _ptr(idx), _ptr(w))
    if rc != 0:
        raise ValueError(f"oracle_route failed ({rc})")
    return logits, idx, w


def permute(topk_idx, E: int, capacity: int = 0) -> dict:
    """Grouping by expert with capacity drop in token order (all int32)."""
    topk_idx = _c(topk_idx, np.int32)
    T, k = topk_idx.shape
    counts = np.empty(E, np.int32)
    dropped = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm_rows = np.empty(T * k, np.int32)
    row_of = np.empty(T * k, np.int32)
    rc = _L().oracle_permute(T, k, E, int(capacity), _ptr(topk_idx), _ptr(counts), _ptr(offsets),
                             _ptr(perm_rows), _ptr(row_of), _ptr(dropped))
    if rc != 0:
        raise ValueError(f"oracle_permute failed ({rc})")
    return dict(counts=counts, offsets=offsets, perm_rows=perm_rows, row_of=row_of.reshape(T, k),
                dropped=dropped)


def moe_tokens(x, w_gate, w_up, w_down, topk_idx, topk_w, dtype: str, row_of=None,
               ws_gate=None, ws_up=None, ws_down=None, tokens=None) -> np.ndarray:
    """fp64 output rows y[t] for the listed tokens (all tokens if None)."""
    x, w_gate, w_up, w_down = _c(x), _c(w_gate), _c(w_up), _c(w_down)
    ws_gate, ws_up, ws_down = _c(ws_gate), _c(ws_up), _c(ws_down)
    topk_idx = _c(topk_idx, np.int32)
    topk_w = _c(topk_w, np.float64)
    row_of = _c(row_of, np.int32)
    T, H = x.shape
    E, I, _ = w_gate.shape
    k = topk_idx.shape[1]
    Is = 0 if ws_gate is None else ws_gate.shape[0]
    tok = None if tokens is None else _c(tokens, np.int32)
    n = T if tok is None else tok.shape[0]
    y = np.empty((n, H), np.float64)
    rc = _L().oracle_moe_tokens(T, H, I, E, k, Is, DTYPE_CODE[dtype], _ptr(x), _ptr(w_gate), _ptr(w_up),
                                _ptr(w_down), _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), _ptr(topk_idx),
                                _ptr(topk_w), _ptr(row_of), n, _ptr(tok), _ptr(y))
    if rc != 0:
        raise ValueError(f"oracle_moe_tokens failed ({rc})")
    return y


def capacity(cf: float, T: int, k: int, E: int) -> int:
    """Per-expert capacity C = ceil(cf * T * k / E), 0 meaning unlimited (cf <= 0).

    The pages name the capacity factor without a formula ("MoE稀疏架构是什么？
    从原理到落地的系统解读", section 三.2; "模型的“分工的艺术”：MoE技术如何提升
    计算效率", section 3.1); the reading taken is the expected share of an
    expert, T * k / E slots, scaled by cf and rounded up.  cf is read as the
    decimal it is written as (the shortest decimal that round-trips the
    Python float, e.g. 1.25 or 0.8) and the product is formed exactly, so no
    binary rounding of cf can lift an exact integer to the next one."""
    from fractions import Fraction

    if cf <= 0:
        return 0
    v = Fraction(repr(float(cf))) * int(T) * int(k) / int(E)
    return int(-((-v.numerator) // v.denominator))  # ceiling of a rational


def topk_margin(logits: np.ndarray, k: int) -> np.ndarray:
    """Gap between the k-th and (k+1)-th largest logit of each token (inf if k == E):
    how far the selection of "MoE稀疏架构是什么？…", section 四 (the k best
    scores) is from changing.  0 for an exact tie across the boundary."""
    T, E = logits.shape
    if k >= E:
        return np.full(T, np.inf)
    part = -np.sort(-logits, axis=1)
    return part[:, k - 1] - part[:, k]


def forward(wl, inp: dict, tokens=None) -> dict:
    """The whole layer for workload ``wl`` (a ``moe_inputs.Workload``).

    Routing and grouping run over all T tokens; the FFN output is evaluated
    for ``tokens`` (all tokens if None).
    """
    logits, idx, w = route(inp["x"], inp["router_w"], inp["router_b"], wl.k, wl.dtype)
    perm = permute(idx, wl.E, capacity(wl.capacity_factor, wl.T, wl.k, wl.E))
    y = moe_tokens(inp["x"], inp["w_gate"], inp["w_up"], inp["w_down"], idx, w, wl.dtype,
                   row_of=perm["row_of"], ws_gate=inp["ws_gate"], ws_up=inp["ws_up"],
                   ws_down=inp["ws_down"], tokens=tokens)
    return dict(logits=logits, topk_idx=idx, topk_w=w, y=y, margin=topk_margin(logits, wl.k), **perm)


def weights_for(logits: np.ndarray, sel: np.ndarray) -> np.ndarray:
    """Softmax over the given selection's scores (fp64), the gating step of
    "MoE稀疏架构是什么？…", section 四 (softmax over the k chosen scores) for
    a selection made elsewhere (a near-tie resolved differently)."""
    l = np.take_along_axis(np.asarray(logits, np.float64), np.asarray(sel, np.int64), 1)
    e = np.exp(l - l.max(1, keepdims=True))
    return e / e.sum(1, keepdims=True)


def expert_rows(x, w_gate, w_up, w_down, tokens, experts, dtype: str) -> np.ndarray:
    """FFN_e(x[t]) (unweighted, fp64) for each (token, expert) pair.  For the
    shared expert pass its weights as [1, Is, H] / [1, H, Is] and expert 0."""
    tokens = np.asarray(tokens, np.int64)
    xs = np.ascontiguousarray(np.asarray(x)[tokens])
    e = np.asarray(experts, np.int32).reshape(-1, 1)
    return moe_tokens(xs, w_gate, w_up, w_down, e, np.ones(e.shape), dtype)


def moe_backward(x, router_w, w_gate, w_up, w_down, topk_idx, topk_w, dy, dtype: str, row_of=None,
                 ws_gate=None, ws_up=None, ws_down=None) -> dict:
    """Gradients of the layer for upstream gradient dy [T, H] (fp64): dx,
    d_router_w, d_router_b, d_w_gate, d_w_up, d_w_down (and d_ws_* with a
    shared expert), by the chain rule through the forward's steps (see
    oracle_moe_backward in moe_oracle.c)."""
    x, router_w, w_gate, w_up, w_down = _c(x), _c(router_w), _c(w_gate), _c(w_up), _c(w_down)
    ws_gate, ws_up, ws_down = _c(ws_gate), _c(ws_up), _c(ws_down)
    topk_idx = _c(topk_idx, np.int32)
    topk_w = _c(topk_w, np.float64)
    row_of = _c(row_of, np.int32)
    dy = _c(dy, np.float64)
    T, H = x.shape
    E, I, _ = w_gate.shape
    k = topk_idx.shape[1]
    Is = 0 if ws_gate is None else ws_gate.shape[0]
    out = dict(dx=np.empty((T, H)), d_router_w=np.empty((E, H)), d_router_b=np.empty(E),
               d_w_gate=np.empty((E, I, H)), d_w_up=np.empty((E, I, H)), d_w_down=np.empty((E, H, I)))
    if Is:
        out.update(d_ws_gate=np.empty((Is, H)), d_ws_up=np.empty((Is, H)), d_ws_down=np.empty((H, Is)))
    rc = _L().oracle_moe_backward(T, H, I, E, k, Is, DTYPE_CODE[dtype], _ptr(x), _ptr(router_w), _ptr(w_gate),
                                  _ptr(w_up), _ptr(w_down), _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down),
                                  _ptr(topk_idx), _ptr(topk_w), _ptr(row_of), _ptr(dy), _ptr(out["dx"]),
                                  _ptr(out["d_router_w"]), _ptr(out["d_router_b"]), _ptr(out["d_w_gate"]),
                                  _ptr(out["d_w_up"]), _ptr(out["d_w_down"]), _ptr(out.get("d_ws_gate")),
                                  _ptr(out.get("d_ws_up")), _ptr(out.get("d_ws_down")))
    if rc != 0:
        raise ValueError(f"oracle_moe_backward failed ({rc})")
    return out


def importance(logits) -> np.ndarray:
    """Per-expert importance: the sum over tokens of the softmax over ALL E
    scores of each token (fp64), the router statistic the load-balance
    penalties start from ("2026年人工智能MoE混合专家模型入门指南", the MoE
    layer's load-balance loss; "模型的“分工的艺术”：MoE技术如何提升计算效率",
    section 3.1, mean gate probability per expert = importance / T).  The
    scores include the router bias."""
    l = np.asarray(logits, np.float64)
    p = np.exp(l - l.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    return p.sum(axis=0)


def balance_losses(importance_e, load_e, T: int) -> dict:
    """The pages' two load-balance penalties from per-expert statistics (fp64).

    kl  -- "模型的“分工的艺术”...", section 3.1: KL(uniform || mean gate
           probability), mean probability q_e = importance_e / T, target
           1/E, log(q_e + 1e-8), and the sum divided by E (the mean over the
           first and only dimension of the E-vector).
    std -- "2026年人工智能MoE...", MoE layer: std(importance) + std(load),
           unbiased standard deviations (divisor E - 1).  load_e is the
           number of tokens whose selection includes e (top-k counts): the
           page's literal load, the number of positive dense-softmax
           probabilities, equals T for every expert.
    switch -- E * sum_e (load_e / T) * (importance_e / T): fraction of tokens
           routed to e times its mean gate probability, the Switch-Transformer
           form (the pages name Switch Transformer's routing in "模型的“分工的
           艺术”...", section 1.2, without a formula).
    """
    imp = np.asarray(importance_e, np.float64)
    load = np.asarray(load_e, np.float64)
    E = imp.size
    q = imp / T
    target = np.full(E, 1.0 / E)
    kl = float(np.sum(target * (np.log(target) - np.log(q + 1e-8))) / E)
    std = float(np.std(imp, ddof=1) + np.std(load, ddof=1))
    switch = float(E * np.sum((load / T) * (imp / T)))
    return dict(kl=kl, std=std, switch=switch)


# ------------------------------------------------------------- mxfp4 weights
# Expert weights in the MXFP4 format of the OCP Microscaling (MX) v1.0
# specification: blocks of 32 elements along the reduction dimension, each
# element an FP4 E2M1 number (sign bit, 2 exponent bits with bias 1, 1
# mantissa bit, subnormal when the exponent field is 0, no inf or NaN) and
# one E8M0 scale per block (value 2^(s - 127); s = 255 is NaN).  The pages
# note that native mxfp4 kernels would speed up gpt-oss ("Mixture of Experts
# (MoEs) in Transformers", section From Dense to Sparse) without giving the
# format; its storage order is read here as two codes per byte, the element
# with the lower index in the low nibble.

def e2m1_value(code: int) -> float:
    """Value of a 4-bit E2M1 code, from its bit fields."""
    sign = -1.0 if code & 0x8 else 1.0
    exp = (code >> 1) & 0x3
    man = code & 0x1
    if exp == 0:
        return sign * (man / 2.0)  # subnormal: 2^(1 - bias) * (m / 2), bias 1
    return sign * 2.0 ** (exp - 1) * (1.0 + man / 2.0)


def mxfp4_dequantize(blocks, scales) -> np.ndarray:
    """float64 weights [..., 32 * nb] from blocks uint8 [..., nb, 16] (two
    codes per byte) and scales uint8 [..., nb]."""
    blocks = np.asarray(blocks, np.uint8)
    scales = np.asarray(scales, np.uint8)
    table = np.array([e2m1_value(c) for c in range(16)], np.float64)
    lo = table[blocks & 0x0F]
    hi = table[blocks >> 4]
    elems = np.stack([lo, hi], axis=-1).reshape(blocks.shape[:-1] + (32,))  # element 2j low, 2j+1 high
    scale = np.where(scales == 255, np.nan, np.ldexp(1.0, scales.astype(np.int64) - 127))
    return (elems * scale[..., None]).reshape(blocks.shape[:-2] + (blocks.shape[-2] * 32,))


def moe_tokens_mxfp4(x, mx: dict, topk_idx, topk_w, dtype: str, row_of=None, tokens=None) -> np.ndarray:
    """moe_tokens with routed experts given as mxfp4 (blocks, scales) pairs
    under "w_gate", "w_up", "w_down".  The dequantized weights and the
    activations are exact in float32 (the scales of the inputs used here
    stay far inside its range), so the fp64 evaluation runs on the exact
    values."""
    w = {}
    for name in ("w_gate", "w_up", "w_down"):
        d = mxfp4_dequantize(*mx[name])
        f = d.astype(np.float32)
        # a scale byte of 255 is NaN (the specification's E8M0 NaN): it
        # propagates to every output that reads the block, as in fp64
        if not np.array_equal(f.astype(np.float64), d, equal_nan=True):
            raise ValueError(f"{name}: mxfp4 values outside the float32 range")
        w[name] = f
    xs = np.asarray(x)
    x32 = _bf16_bits_to_f32(xs) if dtype == "bf16" else xs.astype(np.float32)
    return moe_tokens(x32, w["w_gate"], w["w_up"], w["w_down"], topk_idx, topk_w, "f32", row_of=row_of,
                      tokens=tokens)


def _bf16_bits_to_f32(a) -> np.ndarray:
    """Exact float32 values of bfloat16 bit patterns (uint16)."""
    return (np.asarray(a, np.uint16).astype(np.uint32) << 16).view(np.float32)
