"""Routed MoE FFN layer for B200 (sm_100a): Python binding of ``libmoe.so``.

Every entry point of the C ABI (``include/moe.h``) has a function of the
same name here.  This module only marshals arguments (torch tensors ->
device pointers, the current CUDA stream); every step of the layer runs in
the library's CUDA kernels.  There is no CPU fallback: if the library is
missing or cannot load, calls raise ``MoeError``.

``forward(...)`` is the convenience form of ``moe_forward`` that allocates
the output and the workspace with torch.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_F32, MOE_BF16 = 0, 1
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_CHECK"}
DEVFLAG_BAD_EXPERT_INDEX = 0x1
DEVFLAG_WAIT_TIMEOUT = 0x2


class MoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class moe_config_t(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("top_k", ctypes.c_int32), ("I_shared", ctypes.c_int32),
                ("capacity_factor", ctypes.c_float), ("dtype", ctypes.c_int32)]


class moe_trace_record_t(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("ms", ctypes.c_float)]


_P = ctypes.c_void_p
_SIGS = {
    "moe_workspace_size": ([ctypes.POINTER(moe_config_t)], ctypes.c_size_t),
    "moe_mxfp4_workspace_size": ([ctypes.POINTER(moe_config_t)], ctypes.c_size_t),
    "moe_capacity": ([ctypes.POINTER(moe_config_t)], ctypes.c_int64),
    "moe_route": ([ctypes.POINTER(moe_config_t), _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "moe_route_importance": ([ctypes.POINTER(moe_config_t), _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
                             ctypes.c_int),
    "moe_permute": ([ctypes.POINTER(moe_config_t), _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
                    ctypes.c_int),
    "moe_permute_noalloc": ([ctypes.POINTER(moe_config_t), _P, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "moe_grouped_ffn": ([ctypes.POINTER(moe_config_t)] + [_P] * 11 + [ctypes.c_size_t, _P], ctypes.c_int),
    "moe_combine": ([ctypes.POINTER(moe_config_t), _P, _P, _P, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "moe_forward": ([ctypes.POINTER(moe_config_t)] + [_P] * 14 + [ctypes.c_size_t, _P], ctypes.c_int),
    "moe_forward_routed": ([ctypes.POINTER(moe_config_t)] + [_P] * 14 + [ctypes.c_size_t, _P], ctypes.c_int),
    "moe_shard_capacity_left": ([ctypes.POINTER(moe_config_t), _P, ctypes.c_int32, ctypes.c_int32, _P, _P],
                                ctypes.c_int),
    "moe_shard_capacity_left_host": ([ctypes.POINTER(moe_config_t), _P, ctypes.c_int32, ctypes.c_int32, _P],
                                     ctypes.c_int),
    "moe_balance_losses": ([ctypes.c_int32, ctypes.c_int64, _P, _P, ctypes.POINTER(ctypes.c_double)],
                           ctypes.c_int),
    "moe_forward_expert_shard": ([ctypes.POINTER(moe_config_t), _P, _P, _P, ctypes.c_int32, ctypes.c_int32]
                                 + [_P] * 10 + [ctypes.c_size_t, _P], ctypes.c_int),
    "moe_forward_mxfp4": ([ctypes.POINTER(moe_config_t)] + [_P] * 14 + [ctypes.c_size_t, _P], ctypes.c_int),
    "moe_backward_workspace_size": ([ctypes.POINTER(moe_config_t)], ctypes.c_size_t),
    "moe_backward": ([ctypes.POINTER(moe_config_t)] + [_P] * 21 + [ctypes.c_size_t, _P], ctypes.c_int),
    "moe_reduce_partials": ([ctypes.POINTER(moe_config_t), _P, ctypes.c_int32, _P, _P], ctypes.c_int),
    "moe_get_device_status": ([ctypes.POINTER(moe_config_t), _P, ctypes.c_size_t, _P,
                               ctypes.POINTER(ctypes.c_int32)], ctypes.c_int),
    "moe_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "moe_last_error": ([], ctypes.c_char_p),
    "moe_trace_begin": ([ctypes.c_int32, ctypes.c_char_p], ctypes.c_int),
    "moe_trace_end": ([ctypes.POINTER(moe_trace_record_t), ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)],
                      ctypes.c_int),
}

_lib = None


def load(path: str | None = None):
    """Load libmoe.so (built by ``sparse_mixture_experts_19_b200.build``)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise MoeError(4, f"{p} is missing; build it with `python -m sparse_mixture_experts_19_b200.build`")
    lib = ctypes.CDLL(p)
    for name, (args, res) in _SIGS.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    if path is None:
        _lib = lib
    return lib


def exported_symbols() -> list[str]:
    return list(_SIGS)


def _check(status: int):
    if status != 0:
        raise MoeError(status, load().moe_last_error().decode())


def config(T: int, H: int, I: int, E: int, top_k: int, I_shared: int = 0,
           capacity_factor: float = 0.0, dtype: str = "bf16") -> moe_config_t:
    return moe_config_t(T, H, I, E, top_k, I_shared, capacity_factor,
                        MOE_BF16 if dtype == "bf16" else MOE_F32)


def workspace_size(cfg: moe_config_t) -> int:
    n = load().moe_workspace_size(ctypes.byref(cfg))
    if n == 0:
        raise MoeError(1, load().moe_last_error().decode())
    return n


def capacity(cfg: moe_config_t) -> int:
    return load().moe_capacity(ctypes.byref(cfg))


def _host(a):
    """A host numpy view of a tensor or array (device tensors are copied)."""
    if hasattr(a, "is_cuda"):
        return a.detach().cpu().numpy()
    return a


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise MoeError(1, "tensor is not on a CUDA device")
    if not t.is_contiguous():
        raise MoeError(1, "tensor is not contiguous")
    return t.data_ptr()


def _ws(ws):
    return _ptr(ws), (ws.numel() * ws.element_size() if ws is not None and not isinstance(ws, int) else 0)


def _stream(stream):
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def workspace(cfg: moe_config_t, device="cuda"):
    """A zeroed torch byte tensor big enough for cfg (torch allocations are
    256-byte aligned; zeroed so the device check flags start clear)."""
    import torch

    return torch.zeros(workspace_size(cfg), dtype=torch.uint8, device=device)


def moe_route(cfg, x, router_w, router_b, topk_idx, topk_w, ws, stream=None):
    p, n = _ws(ws)
    _check(load().moe_route(ctypes.byref(cfg), _ptr(x), _ptr(router_w), _ptr(router_b), _ptr(topk_idx),
                            _ptr(topk_w), p, n, _stream(stream)))


def moe_route_importance(cfg, x, router_w, router_b, topk_idx, topk_w, importance, ws, stream=None):
    """moe_route, and the softmax over all E scores of each token added to
    importance [E] float32 (the caller zeroes it)."""
    _check(load().moe_route_importance(ctypes.byref(cfg), _ptr(x), _ptr(router_w), _ptr(router_b),
                                       _ptr(topk_idx), _ptr(topk_w), _ptr(importance), *_ws(ws), _stream(stream)))


def moe_balance_losses(importance, counts, T: int) -> dict:
    """The library's load-balance penalties (kl, std, switch; fp64) from the
    per-expert importance (moe_route_importance) and load (the top-k counts
    from moe_permute or moe_forward) covering T tokens.  Tensors on a device
    are copied to the host first (the C function reads host arrays)."""
    import numpy as np

    imp = np.ascontiguousarray(_host(importance), dtype=np.float32).ravel()
    ld = np.ascontiguousarray(_host(counts), dtype=np.int32).ravel()
    if ld.size != imp.size:
        raise MoeError(1, f"importance has {imp.size} experts, load {ld.size}")
    out = (ctypes.c_double * 3)()
    _check(load().moe_balance_losses(imp.size, int(T), imp.ctypes.data, ld.ctypes.data, out))
    return dict(kl=out[0], std=out[1], switch=out[2])


balance_losses = moe_balance_losses


def moe_permute(cfg, topk_idx, counts, offsets, perm_rows, row_of, dropped, ws, stream=None):
    p, n = _ws(ws)
    _check(load().moe_permute(ctypes.byref(cfg), _ptr(topk_idx), _ptr(counts), _ptr(offsets),
                              _ptr(perm_rows), _ptr(row_of), _ptr(dropped), p, n, _stream(stream)))


def moe_permute_noalloc(cfg, topk_idx, counts, offsets, perm_rows, row_of, dropped, stream=None):
    """moe_permute without a workspace, for callers that cannot allocate device
    memory (allocator callbacks, host-owned memory, allocation-free serving
    loops): the scratch is a fixed static array inside the library.  Limit
    T*top_k <= 1048576; concurrent calls on one device race."""
    _check(load().moe_permute_noalloc(ctypes.byref(cfg), _ptr(topk_idx), _ptr(counts), _ptr(offsets),
                                      _ptr(perm_rows), _ptr(row_of), _ptr(dropped), _stream(stream)))


def moe_grouped_ffn(cfg, x, perm_rows, offsets, w_gate, w_up, w_down, ws_gate, ws_up, ws_down,
                    expert_out, ws, stream=None):
    p, n = _ws(ws)
    _check(load().moe_grouped_ffn(ctypes.byref(cfg), _ptr(x), _ptr(perm_rows), _ptr(offsets), _ptr(w_gate),
                                  _ptr(w_up), _ptr(w_down), _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down),
                                  _ptr(expert_out), p, n, _stream(stream)))


def moe_combine(cfg, expert_out, row_of, topk_w, y, ws, stream=None):
    p, n = _ws(ws)
    _check(load().moe_combine(ctypes.byref(cfg), _ptr(expert_out), _ptr(row_of), _ptr(topk_w), _ptr(y),
                              p, n, _stream(stream)))


def moe_forward(cfg, x, router_w, router_b, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, y,
                topk_idx_out=None, counts_out=None, dropped_out=None, ws=None, stream=None):
    p, n = _ws(ws)
    _check(load().moe_forward(ctypes.byref(cfg), _ptr(x), _ptr(router_w), _ptr(router_b), _ptr(w_gate),
                              _ptr(w_up), _ptr(w_down), _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down), _ptr(y),
                              _ptr(topk_idx_out), _ptr(counts_out), _ptr(dropped_out), p, n,
                              _stream(stream)))


def moe_forward_routed(cfg, x, topk_idx, topk_w, capacity_left, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, y,
                       counts_out=None, dropped_out=None, ws=None, stream=None):
    p, n = _ws(ws)
    _check(load().moe_forward_routed(ctypes.byref(cfg), _ptr(x), _ptr(topk_idx), _ptr(topk_w), _ptr(capacity_left),
                                     _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(ws_gate), _ptr(ws_up),
                                     _ptr(ws_down), _ptr(y), _ptr(counts_out), _ptr(dropped_out), p, n,
                                     _stream(stream)))


def moe_shard_capacity_left(cfg, counts_per_shard, shard: int, capacity_left, stream=None):
    """capacity_left [E] int32 for token shard `shard` of the batch cfg
    describes (cfg.T = tokens of all shards), from every shard's counts
    counts_per_shard [n_shards, E] int32, both on the device."""
    n = counts_per_shard.shape[0]
    _check(load().moe_shard_capacity_left(ctypes.byref(cfg), _ptr(counts_per_shard), n, shard, _ptr(capacity_left),
                                          _stream(stream)))


def moe_shard_capacity_left_host(cfg, counts_per_shard, shard: int):
    """moe_shard_capacity_left on host arrays (counts gathered on the host);
    returns an int32 numpy array [E]."""
    import numpy as np

    c = np.ascontiguousarray(counts_per_shard, dtype=np.int32)
    if c.ndim != 2 or c.shape[1] != cfg.E:
        raise MoeError(1, f"counts_per_shard must be [n_shards, {cfg.E}]")
    out = np.empty(cfg.E, np.int32)
    _check(load().moe_shard_capacity_left_host(ctypes.byref(cfg), c.ctypes.data, c.shape[0], shard,
                                               out.ctypes.data))
    return out


def moe_forward_expert_shard(cfg, x, topk_idx, topk_w, expert_begin: int, expert_count: int, w_gate, w_up, w_down,
                             ws_gate, ws_up, ws_down, y_partial, counts_out=None, dropped_out=None, ws=None,
                             stream=None):
    """This shard's float32 partial output of the layer cfg describes (experts
    [expert_begin, expert_begin + expert_count) held here)."""
    p, n = _ws(ws)
    _check(load().moe_forward_expert_shard(ctypes.byref(cfg), _ptr(x), _ptr(topk_idx), _ptr(topk_w), expert_begin,
                                           expert_count, _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(ws_gate),
                                           _ptr(ws_up), _ptr(ws_down), _ptr(y_partial), _ptr(counts_out),
                                           _ptr(dropped_out), p, n, _stream(stream)))


def moe_forward_mxfp4(cfg, x, router_w, router_b, w_gate_blocks, w_gate_scales, w_up_blocks, w_up_scales,
                      w_down_blocks, w_down_scales, y, topk_idx_out=None, counts_out=None, dropped_out=None, ws=None,
                      stream=None):
    """moe_forward with MXFP4 routed experts (uint8 blocks [E, rows, K/32, 16]
    and scales [E, rows, K/32]).  ws: moe_mxfp4_workspace_size(cfg) bytes
    (mxfp4_workspace); up to 32 routed slots that is moe_workspace_size."""
    p, n = _ws(ws)
    _check(load().moe_forward_mxfp4(ctypes.byref(cfg), _ptr(x), _ptr(router_w), _ptr(router_b), _ptr(w_gate_blocks),
                                    _ptr(w_gate_scales), _ptr(w_up_blocks), _ptr(w_up_scales), _ptr(w_down_blocks),
                                    _ptr(w_down_scales), _ptr(y), _ptr(topk_idx_out), _ptr(counts_out),
                                    _ptr(dropped_out), p, n, _stream(stream)))


def moe_mxfp4_workspace_size(cfg) -> int:
    n = load().moe_mxfp4_workspace_size(ctypes.byref(cfg))
    if n == 0:
        raise MoeError(1, load().moe_last_error().decode())
    return n


def mxfp4_workspace(cfg: moe_config_t, device="cuda"):
    """A zeroed workspace for moe_forward_mxfp4 (see workspace)."""
    import torch

    return torch.zeros(moe_mxfp4_workspace_size(cfg), dtype=torch.uint8, device=device)


def moe_backward_workspace_size(cfg) -> int:
    n = load().moe_backward_workspace_size(ctypes.byref(cfg))
    if n == 0:
        raise MoeError(1, load().moe_last_error().decode())
    return n


def moe_backward(cfg, x, dy, topk_idx, topk_w, router_w, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, dx,
                 d_router_w, d_router_b, d_w_gate, d_w_up, d_w_down, d_ws_gate=None, d_ws_up=None, d_ws_down=None,
                 ws=None, stream=None):
    """Every gradient of the layer (float32 outputs, written) for upstream dy."""
    p, n = _ws(ws)
    _check(load().moe_backward(ctypes.byref(cfg), _ptr(x), _ptr(dy), _ptr(topk_idx), _ptr(topk_w), _ptr(router_w),
                               _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(ws_gate), _ptr(ws_up), _ptr(ws_down),
                               _ptr(dx), _ptr(d_router_w), _ptr(d_router_b), _ptr(d_w_gate), _ptr(d_w_up),
                               _ptr(d_w_down), _ptr(d_ws_gate), _ptr(d_ws_up), _ptr(d_ws_down), p, n,
                               _stream(stream)))


def moe_reduce_partials(cfg, partials, y, stream=None):
    """y = the float32 sum of partials [n, T, H] in order, rounded once."""
    n = 1 if partials.dim() == 2 else partials.shape[0]
    _check(load().moe_reduce_partials(ctypes.byref(cfg), _ptr(partials), n, _ptr(y), _stream(stream)))


def forward_expert_parallel(cfg, x, topk_idx, topk_w, expert_begin: int, expert_count: int, w_gate, w_up, w_down,
                            ws_gate=None, ws_up=None, ws_down=None, group=None, ws=None, stream=None):
    """y on every rank of `group` (torch.distributed, NCCL over NVLink): this
    rank's shard of the experts, an all-reduce of the float32 partial outputs,
    one rounding to the layer dtype."""
    import torch
    import torch.distributed as dist

    T, H = x.shape
    y32 = torch.empty((T, H), dtype=torch.float32, device=x.device)
    if ws is None:
        ws = workspace(cfg, x.device)
    moe_forward_expert_shard(cfg, x, topk_idx, topk_w, expert_begin, expert_count, w_gate, w_up, w_down, ws_gate,
                             ws_up, ws_down, y32, ws=ws, stream=stream)
    dist.all_reduce(y32, group=group)  # the exchange step
    y = torch.empty_like(x)
    moe_reduce_partials(cfg, y32, y, stream)
    return y


def moe_get_device_status(cfg, ws, stream=None) -> int:
    """Waits for the stream; returns the device check flags (and clears them)."""
    p, n = _ws(ws)
    flags = ctypes.c_int32(0)
    st = load().moe_get_device_status(ctypes.byref(cfg), p, n, _stream(stream), ctypes.byref(flags))
    if st not in (0, 5):
        _check(st)
    return flags.value


def moe_status_string(status: int) -> str:
    return load().moe_status_string(status).decode()


def moe_last_error() -> str:
    return load().moe_last_error().decode()


def moe_trace_begin(max_launches: int, only: str | None = None):
    """Trace the next launches (only kernels whose name contains `only`)."""
    _check(load().moe_trace_begin(max_launches, None if only is None else only.encode()))


def moe_trace_end(max_records: int = 4096) -> list[tuple[str, float]]:
    recs = (moe_trace_record_t * max_records)()
    n = ctypes.c_int32(0)
    _check(load().moe_trace_end(recs, max_records, ctypes.byref(n)))
    return [(recs[i].name.decode(), recs[i].ms) for i in range(n.value)]


def forward(x, router_w, w_gate, w_up, w_down, top_k: int, router_b=None, ws_gate=None, ws_up=None,
            ws_down=None, capacity_factor: float = 0.0, ws=None, topk_idx_out=None, counts_out=None,
            dropped_out=None, stream=None):
    """y = MoE(x): the pages' moe_forward(x, experts, router, top_k) on the GPU."""
    import torch

    T, H = x.shape
    E, I, _ = w_gate.shape
    Is = 0 if ws_gate is None else ws_gate.shape[0]
    dtype = "bf16" if x.dtype == torch.bfloat16 else "f32"
    cfg = config(T, H, I, E, top_k, Is, capacity_factor, dtype)
    if ws is None:
        ws = workspace(cfg, x.device)
    y = torch.empty_like(x)
    moe_forward(cfg, x, router_w, router_b, w_gate, w_up, w_down, ws_gate, ws_up, ws_down, y,
                topk_idx_out, counts_out, dropped_out, ws, stream)
    return y
