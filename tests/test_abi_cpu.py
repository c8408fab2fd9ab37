"""CPU-side checks of the C ABI: the library loads, exports every declared symbol, and rejects invalid
arguments before touching the GPU."""
import ctypes
import os
import re

import pytest

from top_expert_selection_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_route.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_list():
    assert declared_symbols() == sorted(B.EXPORTED)


def test_library_exports_every_declared_symbol():
    L = B.lib()
    for name in declared_symbols():
        assert hasattr(L, name), f"{name} missing from {B.LIB_PATH}"


def test_error_strings():
    L = B.lib()
    for code in (0, -1, -2, -3, -4, -5, -6):
        s = L.moe_error_string(code).decode()
        assert s and s != "unknown status"


def _p(**kw):
    base = dict(T=16, E=8, k=2)
    base.update(kw)
    T, E, k = base.pop("T"), base.pop("E"), base.pop("k")
    return B.route_params(T, E, k, **base)


@pytest.mark.parametrize("params,code", [
    (_p(k=9), B.MOE_ERR_INVALID_ARG),                     # k > E
    (_p(k=0), B.MOE_ERR_INVALID_ARG),
    (_p(T=-1), B.MOE_ERR_INVALID_ARG),
    (_p(tile_tokens_dim=6), B.MOE_ERR_INVALID_ARG),       # tile not a power of two
    (_p(score_fn=7), B.MOE_ERR_INVALID_ARG),
    (_p(n_group=3, topk_group=1), B.MOE_ERR_INVALID_ARG),  # groups do not divide E
    (_p(E=16, k=8, n_group=4, topk_group=1), B.MOE_ERR_INVALID_ARG),  # k > topk_group * E / n_group
    (_p(E=16, n_group=4, topk_group=2, group_score_topn=3), B.MOE_ERR_UNSUPPORTED),
    (_p(E=2048, k=2), B.MOE_ERR_UNSUPPORTED),
    (_p(E=64, k=40), B.MOE_ERR_UNSUPPORTED),
    (_p(logits_dtype=5), B.MOE_ERR_INVALID_ARG),
    # expert-parallel shard ranges outside [0, E), or an offset without a count
    (_p(local_expert_offset=-1, local_num_experts=4), B.MOE_ERR_INVALID_ARG),
    (_p(local_expert_offset=6, local_num_experts=4), B.MOE_ERR_INVALID_ARG),
    (_p(local_expert_offset=0, local_num_experts=-2), B.MOE_ERR_INVALID_ARG),
    (_p(local_expert_offset=3, local_num_experts=0), B.MOE_ERR_INVALID_ARG),
    (_p(local_expert_offset=8, local_num_experts=1), B.MOE_ERR_INVALID_ARG),
])
def test_route_validation_rejects_before_any_launch(params, code):
    L = B.lib()
    dummy = ctypes.c_void_p(16)
    args = [dummy] * 11
    rc = L.moe_route(ctypes.byref(params), dummy, None, *args[:9], dummy, ctypes.c_size_t(1 << 20), None)
    assert rc == code
    mp, mt = ctypes.c_int64(), ctypes.c_int64()
    assert L.moe_route_capacity(ctypes.byref(params), ctypes.byref(mp), ctypes.byref(mt)) == code


@pytest.mark.parametrize("off,nl", [(0, 0), (0, 8), (4, 4), (7, 1), (2, 3)])
def test_route_shard_ranges_accepted(off, nl):
    # a valid shard has the single-GPU capacity bound (it never has more rows)
    p = _p(local_expert_offset=off, local_num_experts=nl)
    assert B.route_capacity(p) == B.route_capacity(_p())


def test_route_capacity_formula():
    mp, mt = B.route_capacity(B.route_params(16384, 256, 8, tile_tokens_dim=128))
    assert mp == 16384 * 8 + 256 * 127 and mt == mp // 128
    mp, mt = B.route_capacity(B.route_params(3, 256, 2, tile_tokens_dim=4))
    assert mp == 6 + 6 * 3 and mt == mp // 4


def test_other_entry_points_validate():
    L = B.lib()
    d = ctypes.c_void_p(16)
    sz = ctypes.c_size_t(1 << 20)
    # decode: T > 128 and H % 128 != 0 are page constraints
    assert L.moe_rmsnorm_router_topk(129, 128, 16, 2, 1e-6, 1, d, d, d, None, d, d, d, None, d, sz, None) == -1
    assert L.moe_rmsnorm_router_topk(4, 100, 16, 2, 1e-6, 1, d, d, d, None, d, d, d, None, d, sz, None) == -1
    assert L.moe_rmsnorm_router_topk(4, 128, 24, 2, 1e-6, 1, d, d, d, None, d, d, d, None, d, sz, None) == -2
    assert L.moe_rmsnorm_router_topk(4, 128, 16, 17, 1e-6, 1, d, d, d, None, d, d, d, None, d, sz, None) == -1
    assert L.moe_rmsnorm_router_topk(4, 128, 1040, 8, 1e-6, 1, d, d, d, None, d, d, d, None, d, sz, None) == -2
    nb = ctypes.c_size_t()
    assert L.moe_rmsnorm_router_topk_workspace_bytes(128, 7168, 1024, ctypes.byref(nb)) == 0 and nb.value > 0
    assert L.moe_rmsnorm_router_topk_workspace_bytes(128, 7168, 1040, ctypes.byref(nb)) == -2
    # dispatch / combine: rows must be 16-byte multiples
    assert L.moe_dispatch(4, 3, 2, 1, d, d, d, d, 16, d, None) == -1
    assert L.moe_combine(4, 12, 2, 1, d, 16, d, d, 0, d, None, 0, None) == -1
    assert L.moe_combine(4, 8, 0, 1, d, 16, d, d, 0, d, None, 0, None) == -1
    assert L.moe_combine(4, 8, 2, 1, d, -1, d, d, 0, d, None, 0, None) == -1
    # a status workspace, when given, holds at least the 64-byte header
    assert L.moe_combine(4, 8, 2, 1, d, 16, d, d, 0, d, d, ctypes.c_size_t(8), None) == B.MOE_ERR_WORKSPACE
    # aux
    assert L.moe_aux_scores(4, 8, 9, 0, d, d, d, d, d, sz, None) == -1
    assert L.moe_aux_loss_fwd(4, 0, 8, 2, 0.1, d, d, d, d, sz, None) == -1
    assert L.moe_aux_loss_bwd(4, 4, 8, 0, 0.1, d, d, d, d, d, None) == -1
    # workspace too small
    assert L.moe_aux_scores(4, 8, 2, 0, d, d, d, d, d, ctypes.c_size_t(8), None) == B.MOE_ERR_WORKSPACE
    # wait hook
    assert L.moe_debug_wait_timeout(1, 0, d, sz, None) == -1
    assert L.moe_debug_wait_timeout(1, 10 ** 10, d, sz, None) == -1
    assert L.moe_debug_wait_timeout(1, 1000, d, ctypes.c_size_t(8), None) == B.MOE_ERR_WORKSPACE


def test_fused_shared_experts_validation():
    L = B.lib()
    mp, mt = ctypes.c_int64(), ctypes.c_int64()
    p = B.route_params(16, 8, 2, tile_tokens_dim=4, num_fused_shared_experts=2)
    assert L.moe_route_capacity(ctypes.byref(p), ctypes.byref(mp), ctypes.byref(mt)) == 0
    assert mp.value == 16 * 4 + min(64, 10) * 3 and mt.value == mp.value // 4
    assert L.moe_route_capacity(ctypes.byref(B.route_params(16, 8, 2, num_fused_shared_experts=-1)),
                                ctypes.byref(mp), ctypes.byref(mt)) == B.MOE_ERR_INVALID_ARG
    assert L.moe_route_capacity(ctypes.byref(B.route_params(16, 1020, 2, num_fused_shared_experts=5)),
                                ctypes.byref(mp), ctypes.byref(mt)) == B.MOE_ERR_UNSUPPORTED
    assert L.moe_route_capacity(ctypes.byref(B.route_params(16, 64, 30, num_fused_shared_experts=3)),
                                ctypes.byref(mp), ctypes.byref(mt)) == B.MOE_ERR_UNSUPPORTED


def test_aux_scores_bwd_logits_validates():
    L = B.lib()
    d = ctypes.c_void_p(16)
    assert L.moe_aux_scores_bwd_logits(-1, 8, 0, d, d, d, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_aux_scores_bwd_logits(4, 8, 7, d, d, d, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_aux_scores_bwd_logits(4, 8, 1, None, d, d, None) == B.MOE_ERR_INVALID_ARG
    assert L.moe_aux_scores_bwd_logits(4, 4096, 1, d, d, d, None) == B.MOE_ERR_UNSUPPORTED
    assert L.moe_aux_scores_bwd_logits(0, 8, 1, None, None, None, None) == B.MOE_OK


def test_ep_regroup_validates():
    L = B.lib()
    d = ctypes.c_void_p(16)
    args = lambda W, Lx, H, dt, tile, direction: (W, Lx, H, dt, tile, d, direction, d, 4, d, 16, d, d, d, None, 0, None)
    assert L.moe_ep_regroup(*args(0, 4, 8, 1, 4, 0)) == -1
    assert L.moe_ep_regroup(*args(2, 4, 8, 1, 3, 0)) == -1      # tile not a power of two
    assert L.moe_ep_regroup(*args(2, 4, 4, 1, 4, 0)) == -1      # 8-byte rows
    assert L.moe_ep_regroup(*args(2, 4, 8, 1, 4, 2)) == -1      # no such direction
    assert L.moe_ep_regroup(*args(64, 1024, 8, 1, 4, 0)) == B.MOE_ERR_UNSUPPORTED


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises((ValueError, RuntimeError)):
        B.route(torch.zeros(4, 8), k=2)
