"""The C-ABI library: it loads, exports every symbol include/moe.h declares,
and rejects bad arguments synchronously with status codes (no GPU needed:
every call here returns before anything is enqueued)."""
import ctypes
import os
import re

import numpy as np
import pytest

import sparse_mixture_experts_19_b200 as moe
from sparse_mixture_experts_19_b200 import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return moe.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ("moe_route", "moe_permute", "moe_grouped_ffn", "moe_combine", "moe_forward",
              "moe_workspace_size"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert sorted(names) == sorted(moe.exported_symbols())
    for n in names:
        assert hasattr(lib, n), n


def test_binding_signatures_match_the_header():
    """Every declared function's ctypes argtypes has as many entries as the
    header's parameter list: an argument past the argtypes would be converted
    by ctypes' defaults (a Python int becomes a 32-bit C int), so a 64-bit
    parameter there (the stream) would arrive with garbage upper bits."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    decls = re.findall(r"\b(moe_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S)
    assert decls
    for name, params in decls:
        params = params.strip()
        n = 0 if params in ("", "void") else len([q for q in params.split(",") if q.strip()])
        assert len(moe._SIGS[name][0]) == n, f"{name}: header has {n} parameters, binding {len(moe._SIGS[name][0])}"


def cfg(**kw):
    base = dict(T=64, H=128, I=256, E=8, top_k=2, I_shared=0, capacity_factor=0.0, dtype="bf16")
    base.update(kw)
    return moe.config(**base)


@pytest.mark.parametrize("bad", [
    dict(T=-1), dict(H=0), dict(H=12), dict(I=4), dict(E=0), dict(E=257), dict(top_k=0),
    dict(top_k=9, E=16), dict(top_k=3, E=2), dict(I_shared=6), dict(capacity_factor=float("nan")),
])
def test_invalid_configs_have_no_workspace(lib, bad):
    assert lib.moe_workspace_size(ctypes.byref(cfg(**bad))) == 0
    assert moe.moe_last_error()


def test_dense_top_k_equal_E_allowed_up_to_32(lib):
    assert lib.moe_workspace_size(ctypes.byref(cfg(E=16, top_k=16))) > 0
    assert lib.moe_workspace_size(ctypes.byref(cfg(E=33, top_k=33))) == 0


def test_workspace_size_grows_with_tokens(lib):
    a = lib.moe_workspace_size(ctypes.byref(cfg(T=64)))
    b = lib.moe_workspace_size(ctypes.byref(cfg(T=1000)))
    assert 0 < a < b
    assert a % 256 == 0


def test_capacity(lib):
    c = moe.config(32768, 2048, 768, 128, 8, 0, 1.25, "bf16")
    assert moe.capacity(c) == 2560
    assert moe.capacity(cfg()) == 0


FAKE = 0x7f0000000000  # never dereferenced: every call below fails validation first


def call_forward(lib, c, ws, ws_bytes, **ptrs):
    p = dict(x=FAKE, router_w=FAKE, router_b=None, w_gate=FAKE, w_up=FAKE, w_down=FAKE,
             ws_gate=None, ws_up=None, ws_down=None, y=FAKE)
    p.update(ptrs)
    return lib.moe_forward(ctypes.byref(c), p["x"], p["router_w"], p["router_b"], p["w_gate"], p["w_up"],
                           p["w_down"], p["ws_gate"], p["ws_up"], p["ws_down"], p["y"], None, None, None,
                           ws, ws_bytes, None)


def test_forward_rejects_small_or_misaligned_workspace(lib):
    c = cfg()
    need = lib.moe_workspace_size(ctypes.byref(c))
    assert call_forward(lib, c, FAKE, need - 1) == 3
    assert "needs" in moe.moe_last_error()
    assert call_forward(lib, c, FAKE + 16, need) == 3
    assert call_forward(lib, c, None, need) == 3


@pytest.mark.parametrize("field", ["x", "router_w", "w_gate", "w_up", "w_down", "y"])
def test_forward_rejects_null_and_misaligned_pointers(lib, field):
    c = cfg()
    need = lib.moe_workspace_size(ctypes.byref(c))
    assert call_forward(lib, c, FAKE, need, **{field: None}) == 1
    assert field in moe.moe_last_error()
    assert call_forward(lib, c, FAKE, need, **{field: FAKE + 2}) == 1


def test_forward_requires_shared_weights_when_configured(lib):
    c = cfg(I_shared=64)
    need = lib.moe_workspace_size(ctypes.byref(c))
    assert call_forward(lib, c, FAKE, need) == 1
    assert call_forward(lib, c, FAKE, need, ws_gate=FAKE, ws_up=FAKE, ws_down=FAKE + 4) == 1


def test_forward_with_no_tokens_is_a_no_op(lib):
    c = cfg(T=0)
    need = lib.moe_workspace_size(ctypes.byref(c))
    assert call_forward(lib, c, FAKE, need, x=None, y=None) == 0


def test_stage_calls_validate(lib):
    c = cfg()
    need = lib.moe_workspace_size(ctypes.byref(c))
    assert lib.moe_route(None, FAKE, FAKE, None, FAKE, FAKE, FAKE, need, None) == 1
    assert lib.moe_route(ctypes.byref(c), FAKE, FAKE, FAKE + 4, FAKE, FAKE, FAKE, need, None) == 1
    assert lib.moe_permute(ctypes.byref(c), FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, need, None) == 1
    assert lib.moe_grouped_ffn(ctypes.byref(c), FAKE, FAKE, FAKE, FAKE, FAKE, None, None, None, None, FAKE,
                               FAKE, need, None) == 1
    assert lib.moe_combine(ctypes.byref(c), FAKE, FAKE, FAKE, None, FAKE, need, None) == 1


def test_route_importance_validates(lib):
    c = cfg(T=300, E=16, top_k=4)
    need = lib.moe_workspace_size(ctypes.byref(c))

    def call(**kw):
        p = dict(x=FAKE, router_w=FAKE, router_b=None, topk_idx=FAKE, topk_w=FAKE, importance=FAKE)
        p.update(kw)
        return lib.moe_route_importance(ctypes.byref(c), p["x"], p["router_w"], p["router_b"],
                                        p["topk_idx"], p["topk_w"], p["importance"], FAKE, need, None)

    assert call(importance=None) == 1 and "importance" in moe.moe_last_error()
    assert call(importance=FAKE + 4) == 1
    for field in ("x", "router_w", "topk_idx", "topk_w"):
        assert call(**{field: None}) == 1 and field in moe.moe_last_error()
    assert call(router_b=FAKE + 8) == 1
    c0 = cfg(T=0, E=16, top_k=4)
    assert lib.moe_route_importance(ctypes.byref(c0), None, None, None, None, None, FAKE, FAKE, need, None) == 0


def test_balance_losses_call_matches_oracle():
    """moe_balance_losses (host C, fp64) against the oracle's penalties on the
    same float32 importance."""
    import oracle
    rng = np.random.default_rng(11)
    for E, T in ((2, 10), (8, 1000), (256, 16384)):
        imp = (rng.dirichlet(np.ones(E)) * T).astype(np.float32)
        load = rng.integers(0, 8 * T // E + 1, E).astype(np.int32)
        got = moe.moe_balance_losses(imp, load, T)
        ref = oracle.balance_losses(imp.astype(np.float64), load, T)
        for key in ("kl", "std", "switch"):
            assert abs(got[key] - ref[key]) <= 1e-12 * max(1.0, abs(ref[key])), (E, key)
    with pytest.raises(moe.MoeError):
        moe.moe_balance_losses(np.ones(1), np.ones(1), 4)
    with pytest.raises(moe.MoeError):
        moe.moe_balance_losses(np.ones(4), np.ones(4), 0)
    with pytest.raises(moe.MoeError):
        moe.moe_balance_losses(np.ones(4), np.ones(3), 4)


def test_shard_capacity_left_validates(lib):
    c = cfg(capacity_factor=1.0)
    assert lib.moe_shard_capacity_left(ctypes.byref(c), FAKE, 2, 2, FAKE, None) == 1
    assert lib.moe_shard_capacity_left(ctypes.byref(c), FAKE, 0, 0, FAKE, None) == 1
    assert lib.moe_shard_capacity_left(ctypes.byref(c), None, 2, 1, FAKE, None) == 1
    assert lib.moe_shard_capacity_left(ctypes.byref(cfg()), FAKE, 2, 1, FAKE, None) == 1
    assert "capacity" in moe.moe_last_error()


def call_forward_routed(lib, c, ws, ws_bytes, **ptrs):
    p = dict(x=FAKE, topk_idx=FAKE, topk_w=FAKE, capacity_left=None, w_gate=FAKE, w_up=FAKE, w_down=FAKE,
             ws_gate=None, ws_up=None, ws_down=None, y=FAKE)
    p.update(ptrs)
    return lib.moe_forward_routed(ctypes.byref(c), p["x"], p["topk_idx"], p["topk_w"], p["capacity_left"],
                                  p["w_gate"], p["w_up"], p["w_down"], p["ws_gate"], p["ws_up"], p["ws_down"],
                                  p["y"], None, None, ws, ws_bytes, None)


@pytest.mark.parametrize("field", ["x", "topk_idx", "topk_w", "w_gate", "w_up", "w_down", "y"])
def test_forward_routed_rejects_null_and_misaligned_pointers(lib, field):
    c = cfg(capacity_factor=1.0)
    need = lib.moe_workspace_size(ctypes.byref(c))
    assert call_forward_routed(lib, c, FAKE, need, **{field: None}) == 1
    assert field in moe.moe_last_error()
    assert call_forward_routed(lib, c, FAKE, need, **{field: FAKE + 4}) == 1


def test_forward_routed_optional_capacity_must_be_aligned(lib):
    c = cfg(capacity_factor=1.0)
    need = lib.moe_workspace_size(ctypes.byref(c))
    assert call_forward_routed(lib, c, FAKE, need, capacity_left=FAKE + 8) == 1
    assert "capacity_left" in moe.moe_last_error()
    assert call_forward_routed(lib, c, FAKE, need - 1) == 3
    assert call_forward_routed(lib, cfg(T=0), FAKE, need, x=None, y=None) == 0


def test_capacity_ceiling_ignores_float32_rounding_of_the_factor(lib):
    # 0.8 is stored as 0.800000012 in float32; 0.8 * 1200 * 2 / 8 = 240 exactly
    assert moe.capacity(cfg(T=1200, E=8, top_k=2, capacity_factor=0.8)) == 240
    assert moe.capacity(cfg(T=1201, E=8, top_k=2, capacity_factor=0.8)) == 241
    assert moe.capacity(cfg(T=3000, E=128, top_k=8, capacity_factor=1.25)) == 235


def test_status_strings(lib):
    for code, name in moe.STATUS.items():
        assert moe.moe_status_string(code) == name
    assert moe.moe_status_string(99) == "MOE_ERR_UNKNOWN"


def test_trace_end_without_begin_fails(lib):
    with pytest.raises(moe.MoeError):
        moe.moe_trace_end()


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.dirname(moe.__file__)
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(root, f), encoding="utf-8").read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "moe_oracle" not in src, f


def test_missing_library_raises_instead_of_falling_back(tmp_path):
    with pytest.raises(moe.MoeError) as e:
        moe.load(str(tmp_path / "libmoe.so"))
    assert "missing" in str(e.value)
