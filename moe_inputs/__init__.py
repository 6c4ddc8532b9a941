"""Seeded synthetic inputs for the routed MoE FFN layer.

This module is shared by the CUDA path's tests/bench and by the CPU oracle.
It holds no arithmetic of the MoE method: it only describes the workloads
(shapes and the input recipe) and produces their input bytes from a
counter-based generator (splitmix64 + Box-Muller, see ``gen.c``).

Input recipe (every workload):
  * x ~ N(0, 1); router weights ``router_w [E, H]`` ~ N(0, 1/H);
    ``w_gate``, ``w_up [E, I, H]`` ~ N(0, 1/H); ``w_down [E, H, I]`` ~ N(0, 1/I);
    shared expert (when present) likewise with I_s.
  * Values are drawn in double, rounded to float32 and, for bf16 workloads,
    to bfloat16 (round to nearest even).  Arrays of a bf16 workload are
    returned as ``uint16`` bit patterns.
  * Zipf-skewed routing: ``router_b[e] = -s * ln(rank_e)`` with ``rank`` a
    seeded permutation of 1..E, so exp(b_e), the prior weight of expert e in
    the softmax, is proportional to rank_e^-s (a Zipf(s) popularity law).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libmoe_inputs.so")

# stream ids: one independent stream per tensor
STREAM_X = 1
STREAM_ROUTER_W = 2
STREAM_W_GATE = 3
STREAM_W_UP = 4
STREAM_W_DOWN = 5
STREAM_WS_GATE = 6
STREAM_WS_UP = 7
STREAM_WS_DOWN = 8
STREAM_ZIPF_RANK = 9
STREAM_SAMPLE = 10
STREAM_MX_GATE, STREAM_MX_UP, STREAM_MX_DOWN = 11, 12, 13        # mxfp4 element codes
STREAM_MXS_GATE, STREAM_MXS_UP, STREAM_MXS_DOWN = 14, 15, 16     # mxfp4 block scales


def build(force: bool = False) -> str:
    """Compile gen.c into libmoe_inputs.so (gcc, OpenMP)."""
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
        u64, i64 = ctypes.c_uint64, ctypes.c_int64
        _lib.moe_gen_normal_f32.argtypes = [u64, u64, u64, i64, ctypes.c_double, ctypes.c_void_p]
        _lib.moe_gen_normal_bf16.argtypes = [u64, u64, u64, i64, ctypes.c_double, ctypes.c_void_p]
        _lib.moe_gen_permutation.argtypes = [u64, u64, ctypes.c_int32, ctypes.c_void_p]
        _lib.moe_gen_bytes.argtypes = [u64, u64, u64, i64, ctypes.c_void_p]
        _lib.moe_gen_u64.argtypes = [u64, u64, u64]
        _lib.moe_gen_u64.restype = u64
    return _lib


def normal(seed: int, stream: int, shape, std: float, dtype: str, first: int = 0) -> np.ndarray:
    """Elements [first, first+n) of stream (seed, stream), scaled by std.

    dtype "f32" -> float32 array; "bf16" -> uint16 array of bfloat16 bits.
    """
    n = int(np.prod(shape)) if len(shape) else 1
    if dtype == "f32":
        out = np.empty(shape, dtype=np.float32)
        _L().moe_gen_normal_f32(seed, stream, first, n, std, out.ctypes.data)
    elif dtype == "bf16":
        out = np.empty(shape, dtype=np.uint16)
        _L().moe_gen_normal_bf16(seed, stream, first, n, std, out.ctypes.data)
    else:
        raise ValueError(dtype)
    return out


def permutation(seed: int, stream: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    _L().moe_gen_permutation(seed, stream, n, out.ctypes.data)
    return out


def random_bytes(seed: int, stream: int, shape, first: int = 0) -> np.ndarray:
    """Uniform random bytes [first, first+n) of stream (seed, stream)."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(shape, dtype=np.uint8)
    _L().moe_gen_bytes(seed, stream, first, n, out.ctypes.data)
    return out


def mxfp4_weights(seed: int, code_stream: int, scale_stream: int, E: int, rows: int, cols: int,
                  fan_in: int) -> tuple:
    """Synthetic mxfp4 expert weights [E, rows, cols] (blocks of 32 along
    cols): uniformly random 4-bit element codes, two per byte, and one scale
    byte per block, drawn from the three exponents around the one that gives
    weights of RMS about 1/sqrt(fan_in) (uniform codes have an RMS magnitude
    of about 2.93; scale byte s stands for 2^(s - 127)).  Returns
    (blocks uint8 [E, rows, cols/32, 16], scales uint8 [E, rows, cols/32])."""
    if cols % 32:
        raise ValueError("cols must be a multiple of 32")
    nb = cols // 32
    blocks = random_bytes(seed, code_stream, (E, rows, nb, 16))
    center = 127 + int(round(math.log2(1.0 / (math.sqrt(fan_in) * 2.926))))
    scales = (center - 1 + random_bytes(seed, scale_stream, (E, rows, nb)) % 3).astype(np.uint8)
    return blocks, scales


def make_mxfp4_experts(w: "Workload") -> dict:
    """mxfp4 versions of the routed experts of workload w (gate/up [E, I, H],
    down [E, H, I]), as (blocks, scales) pairs; H and I multiples of 32."""
    s = w.seed
    return {
        "w_gate": mxfp4_weights(s, STREAM_MX_GATE, STREAM_MXS_GATE, w.E, w.I, w.H, w.H),
        "w_up": mxfp4_weights(s, STREAM_MX_UP, STREAM_MXS_UP, w.E, w.I, w.H, w.H),
        "w_down": mxfp4_weights(s, STREAM_MX_DOWN, STREAM_MXS_DOWN, w.E, w.H, w.I, w.I),
    }


def u64(seed: int, stream: int, n: int) -> int:
    return int(_L().moe_gen_u64(seed, stream, n))


def sample_tokens(seed: int, T: int, n: int) -> np.ndarray:
    """A seeded, sorted sample of n distinct token ids out of range(T)."""
    if n >= T:
        return np.arange(T, dtype=np.int32)
    perm = permutation(seed, STREAM_SAMPLE, T)
    return np.sort(perm[:n]).astype(np.int32)


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (a.astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class Workload:
    """One MoE-layer workload: shapes plus input recipe."""

    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    dtype: str = "bf16"          # "f32" or "bf16"
    I_shared: int = 0            # 0 = no shared expert
    capacity_factor: float = 0.0  # <= 0: no capacity limit
    zipf_s: float = 0.0          # > 0: router bias b_e = -s ln(rank_e)
    seed: int = 0
    note: str = ""

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def has_bias(self) -> bool:
        return self.zipf_s > 0


# The five workload families (full sizes).
TINY = Workload("tiny_f32", T=64, H=128, I=256, E=8, k=2, dtype="f32",
                note="tiny MoE layer, fp32, near-uniform routing")
MIXTRAL = Workload("mixtral_8x7b_layer", T=4096, H=4096, I=14336, E=8, k=2,
                   note="Mixtral-8x7B-shaped layer, near-uniform routing")
GPTOSS = Workload("gpt_oss_20b_layer", T=8192, H=2880, I=2880, E=32, k=4,
                  note="gpt-oss-20b-shaped layer; T swept over 1, 8, 64, 512, 8192")
GPTOSS_T = (1, 8, 64, 512, 8192)
FINE = Workload("fine_grained_e256_layer", T=16384, H=7168, I=2048, E=256, k=8, I_shared=2048,
                zipf_s=1.1, note="256 routed experts top-8 + 1 shared expert, Zipf(1.1) router bias")
QWEN3 = Workload("qwen3_30b_a3b_layer", T=32768, H=2048, I=768, E=128, k=8, capacity_factor=1.25,
                 note="Qwen3-30B-A3B-shaped layer, capacity factor 1.25, overflow dropped in token order")

FULL = {w.name: w for w in (TINY, MIXTRAL, GPTOSS, FINE, QWEN3)}

# Reduced variants: same routing structure (E, k, bias, capacity factor),
# smaller H/I/T so the oracle finishes in seconds, with ragged tails.
SMALL = {
    "tiny_f32": TINY,
    "mixtral_8x7b_layer": MIXTRAL.with_(name="mixtral_small", T=1000, H=512, I=1792),
    "gpt_oss_20b_layer": GPTOSS.with_(name="gpt_oss_small", T=777, H=576, I=576),
    "fine_grained_e256_layer": FINE.with_(name="fine_small", T=1500, H=512, I=256, I_shared=256),
    "qwen3_30b_a3b_layer": QWEN3.with_(name="qwen3_small", T=3000, H=512, I=384),
}


def make_inputs(w: Workload, router_only: bool = False) -> dict:
    """All inputs of workload w as numpy arrays (bf16 as uint16 bits).

    router_only: only x, router_w and router_b (expert weights are None)."""
    s, dt = w.seed, w.dtype
    out = {
        "x": normal(s, STREAM_X, (w.T, w.H), 1.0, dt),
        "router_w": normal(s, STREAM_ROUTER_W, (w.E, w.H), 1.0 / math.sqrt(w.H), dt),
        "w_gate": None, "w_up": None, "w_down": None,
        "router_b": None,
        "ws_gate": None, "ws_up": None, "ws_down": None,
    }
    if w.has_bias:
        rank = permutation(s, STREAM_ZIPF_RANK, w.E).astype(np.float64) + 1.0
        out["router_b"] = (-w.zipf_s * np.log(rank)).astype(np.float32)
    if router_only:
        return out
    out["w_gate"] = normal(s, STREAM_W_GATE, (w.E, w.I, w.H), 1.0 / math.sqrt(w.H), dt)
    out["w_up"] = normal(s, STREAM_W_UP, (w.E, w.I, w.H), 1.0 / math.sqrt(w.H), dt)
    out["w_down"] = normal(s, STREAM_W_DOWN, (w.E, w.H, w.I), 1.0 / math.sqrt(w.I), dt)
    if w.I_shared > 0:
        Is = w.I_shared
        out["ws_gate"] = normal(s, STREAM_WS_GATE, (Is, w.H), 1.0 / math.sqrt(w.H), dt)
        out["ws_up"] = normal(s, STREAM_WS_UP, (Is, w.H), 1.0 / math.sqrt(w.H), dt)
        out["ws_down"] = normal(s, STREAM_WS_DOWN, (w.H, Is), 1.0 / math.sqrt(Is), dt)
    return out
