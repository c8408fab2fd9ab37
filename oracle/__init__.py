"""CPU oracle for the MoE routing path -- TEST INFRASTRUCTURE ONLY.

A ctypes wrapper over ``oracle.c`` (plain single-threaded C, fp32 where the
method fixes fp32, double where a plain sum is the definition).  Only the test
suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package.  It shares no code with the CUDA library and never calls
it.

Arrays are numpy; bf16 tensors travel as their raw uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

F32 = 0
BF16 = 1
SOFTMAX = 0
SIGMOID = 1

_lib_handle = None


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (gcc, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
                               "-Wall", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _lib():
    global _lib_handle
    if _lib_handle is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32 = ctypes.c_int
        f32 = ctypes.c_float
        L.oracle_route_select.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, i32, f32,
                                          P, i32, P, i32, P, P, P, P, P]
        L.oracle_route_capacity.argtypes = [i32, i32, i32, i32, P, P]
        L.oracle_route_bookkeeping.argtypes = [i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P]
        L.oracle_route_bookkeeping_shared.argtypes = [i32, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P]
        L.oracle_append_shared.argtypes = [i32, i32, i32, i32, P, P, P, P]
        L.oracle_aux_scores.argtypes = [i32, i32, i32, i32, P, P, P, P]
        L.oracle_aux_loss_fwd.argtypes = [i32, i32, i32, i32, f32, P, P, P]
        L.oracle_aux_loss_bwd.argtypes = [i32, i32, i32, i32, f32, f32, P, P, P, P]
        L.oracle_aux_scores_bwd.argtypes = [i32, i32, i32, P, P, P]
        L.oracle_aux_scores_bwd_logits.argtypes = [i32, i32, i32, P, P, P]
        L.oracle_route_weights_bwd.argtypes = [i32, i32, i32, i32, i32, i32, f32, P, P, P, P]
        L.oracle_dispatch.argtypes = [i32, i32, i32, P, P, P, i32, P]
        L.oracle_combine.argtypes = [i32, i32, i32, P, P, P, i32, P]
        L.oracle_combine_f32.argtypes = [i32, i32, i32, P, P, P, i32, P]
        L.oracle_ep_regroup.argtypes = [i32, i32, i32, P, P, ctypes.c_longlong, ctypes.c_longlong, P, P, P, P]
        L.oracle_rmsnorm_router_topk.argtypes = [i32, i32, i32, i32, f32, i32, P, P, P, P, P, P, P, P]
        L.oracle_router_logits.argtypes = [i32, i32, i32, P, P, P, P]
        L.oracle_router_logits.restype = i32
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f32.restype = f32
        L.oracle_f32_to_bf16.argtypes = [f32]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
        L.oracle_f64_to_bf16.restype = ctypes.c_uint16
        for name in ("oracle_route_select", "oracle_route_capacity", "oracle_route_bookkeeping",
                     "oracle_route_bookkeeping_shared", "oracle_append_shared",
                     "oracle_aux_scores", "oracle_aux_loss_fwd", "oracle_aux_loss_bwd", "oracle_aux_scores_bwd", "oracle_aux_scores_bwd_logits",
                     "oracle_route_weights_bwd",
                     "oracle_dispatch", "oracle_combine", "oracle_combine_f32", "oracle_ep_regroup", "oracle_rmsnorm_router_topk"):
            getattr(L, name).restype = i32
        _lib_handle = L
    return _lib_handle


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def as_numpy(x, dtype_code: Optional[int] = None) -> np.ndarray:
    """torch CPU tensor or numpy array -> contiguous numpy (bf16 as uint16 bits)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16).copy()
            return x.numpy().copy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(x)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float32:
        return F32
    raise TypeError(f"unsupported dtype {a.dtype}")


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"{what}: invalid argument (oracle rc={rc})")


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    """Elementwise bf16 bits -> fp32 through the oracle's own conversion."""
    L = _lib()
    flat = np.asarray(a, dtype=np.uint16).ravel()
    return np.array([L.oracle_bf16_to_f32(int(v)) for v in flat], dtype=np.float32).reshape(np.shape(a))


def f32_to_bf16(a: np.ndarray) -> np.ndarray:
    L = _lib()
    flat = np.asarray(a, dtype=np.float32).ravel()
    return np.array([L.oracle_f32_to_bf16(float(v)) for v in flat], dtype=np.uint16).reshape(np.shape(a))


def f64_to_bf16(a: np.ndarray) -> np.ndarray:
    L = _lib()
    flat = np.asarray(a, dtype=np.float64).ravel()
    return np.array([L.oracle_f64_to_bf16(float(v)) for v in flat], dtype=np.uint16).reshape(np.shape(a))


def route_select(logits, *, k: int, score_fn: int = SOFTMAX, softmax_before_topk: int = 1,
                 n_group: int = 0, topk_group: int = 0, group_score_topn: int = 2,
                 renormalize: int = 1, scaling_factor: float = 1.0, bias=None) -> dict:
    lg = as_numpy(logits)
    T, E = lg.shape
    b = as_numpy(bias) if bias is not None else None
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    keys = np.zeros((T, E), np.float32)
    G = max(n_group, 1)
    gsc = np.zeros((T, G), np.float32)
    gkept = np.zeros((T, G), np.uint8)
    rc = _lib().oracle_route_select(T, E, k, score_fn, softmax_before_topk, n_group, topk_group,
                                    group_score_topn, renormalize, float(scaling_factor),
                                    _ptr(lg), _dtype_code(lg), _ptr(b),
                                    _dtype_code(b) if b is not None else F32,
                                    _ptr(ids), _ptr(w), _ptr(keys), _ptr(gsc), _ptr(gkept))
    _check(rc, "route_select")
    return {"ids": ids, "weights": w, "keys": keys, "group_scores": gsc, "group_kept": gkept}


def route_capacity(T: int, E: int, k: int, tile: int):
    mp = ctypes.c_int64()
    mt = ctypes.c_int64()
    rc = _lib().oracle_route_capacity(T, E, k, tile, ctypes.byref(mp), ctypes.byref(mt))
    _check(rc, "route_capacity")
    return int(mp.value), int(mt.value)


def route_bookkeeping(ids, E: int, tile: int, local_expert_offset: int = 0,
                      local_num_experts: Optional[int] = None, num_shared: int = 0) -> dict:
    """Bookkeeping of the experts [local_expert_offset, local_expert_offset + local_num_experts)
    (all E by default) and of the num_shared fused shared experts E .. E + num_shared - 1 (local
    index local_num_experts + s); counts/offsets/tile_expert are indexed by the local expert."""
    ids = as_numpy(ids).astype(np.int32, copy=False)
    T, k = ids.shape
    nl = E if local_num_experts is None else int(local_num_experts)
    NL = nl + num_shared
    rows = T * k
    max_padded = rows + min(rows, E + num_shared) * (tile - 1)
    max_tiles = max_padded // tile
    counts = np.zeros(NL, np.int32)
    offsets = np.zeros(NL + 1, np.int32)
    e2p = np.zeros(T * k, np.int32)
    p2t = np.full(max(max_padded, 1), -7, np.int32)
    te = np.full(max(max_tiles, 1), -7, np.int32)
    tl = np.full(max(max_tiles, 1), -7, np.int32)
    totals = np.zeros(2, np.int32)
    rc = _lib().oracle_route_bookkeeping_shared(T, E, num_shared, k, tile, int(local_expert_offset), nl,
                                                _ptr(np.ascontiguousarray(ids)), _ptr(counts), _ptr(offsets),
                                                _ptr(e2p), _ptr(p2t), _ptr(te), _ptr(tl), _ptr(totals))
    _check(rc, "route_bookkeeping")
    P, nt = int(totals[0]), int(totals[1])
    return {"counts": counts, "offsets": offsets, "e2p": e2p, "p2t": p2t[:P], "tile_expert": te[:nt],
            "tile_mn_limit": tl[:nt], "totals": totals, "max_padded": max_padded, "max_tiles": max_tiles}


def append_shared(ids, weights, E: int, S: int):
    """The S fused shared-expert slots appended to each token: ids E + s, weights 1.0."""
    ids = np.ascontiguousarray(as_numpy(ids), dtype=np.int32)
    w = np.ascontiguousarray(as_numpy(weights), dtype=np.float32)
    T, k = ids.shape
    io = np.zeros((T, k + S), np.int32)
    wo = np.zeros((T, k + S), np.float32)
    _check(_lib().oracle_append_shared(T, k, S, E, _ptr(ids), _ptr(w), _ptr(io), _ptr(wo)), "append_shared")
    return io, wo


def aux_scores(logits, k: int, score_fn: int = SOFTMAX) -> dict:
    lg = as_numpy(logits).astype(np.float32, copy=False)
    T, E = lg.shape
    probs = np.zeros((T, E), np.float32)
    rmap = np.zeros((T, E), np.uint8)
    tpe = np.zeros(E, np.int32)
    rc = _lib().oracle_aux_scores(T, E, k, score_fn, _ptr(np.ascontiguousarray(lg)), _ptr(probs),
                                  _ptr(rmap), _ptr(tpe))
    _check(rc, "aux_scores")
    return {"probs": probs, "routing_map": rmap, "tokens_per_expert": tpe}


def aux_loss_fwd(probs, tokens_per_expert, T_total: int, k: int, coeff: float) -> float:
    p = np.ascontiguousarray(as_numpy(probs), dtype=np.float32)
    tpe = np.ascontiguousarray(as_numpy(tokens_per_expert), dtype=np.int32)
    T, E = p.shape
    out = np.zeros(1, np.float32)
    rc = _lib().oracle_aux_loss_fwd(T, T_total, E, k, float(coeff), _ptr(p), _ptr(tpe), _ptr(out))
    _check(rc, "aux_loss_fwd")
    return float(out[0])


def aux_loss_bwd(probs, tokens_per_expert, T_total: int, k: int, coeff: float, grad_loss: float) -> dict:
    p = np.ascontiguousarray(as_numpy(probs), dtype=np.float32)
    tpe = np.ascontiguousarray(as_numpy(tokens_per_expert), dtype=np.int32)
    T, E = p.shape
    gp = np.zeros((T, E), np.float32)
    gl = np.zeros((T, E), np.float32)
    rc = _lib().oracle_aux_loss_bwd(T, T_total, E, k, float(coeff), float(grad_loss), _ptr(p), _ptr(tpe),
                                    _ptr(gp), _ptr(gl))
    _check(rc, "aux_loss_bwd")
    return {"grad_probs": gp, "grad_logits": gl}


def route_weights_bwd(logits, ids, grad_weights, *, score_fn: int, softmax_before_topk: int = 1,
                      renormalize: int = 1, scaling_factor: float = 1.0) -> np.ndarray:
    """dL/dlogits [T,E] for the routed weights of the given selection (fp32 logits)."""
    lg = np.ascontiguousarray(as_numpy(logits), dtype=np.float32)
    idv = np.ascontiguousarray(as_numpy(ids), dtype=np.int32)
    gw = np.ascontiguousarray(as_numpy(grad_weights), dtype=np.float32)
    T, E = lg.shape
    k = idv.shape[1]
    gl = np.zeros((T, E), np.float32)
    _check(_lib().oracle_route_weights_bwd(T, E, k, int(score_fn), int(softmax_before_topk), int(renormalize),
                                           float(scaling_factor), _ptr(lg), _ptr(idv), _ptr(gw), _ptr(gl)),
           "route_weights_bwd")
    return gl


def aux_scores_bwd_logits(logits, grad_probs, score_fn: int = 0) -> np.ndarray:
    """dL/dlogits of the aux scores (softmax, or sigmoid over the row sum) given dL/dprobs, the scores
    recomputed from the logits."""
    x = np.ascontiguousarray(as_numpy(logits), dtype=np.float32)
    g = np.ascontiguousarray(as_numpy(grad_probs), dtype=np.float32)
    T, E = x.shape
    gl = np.zeros((T, E), np.float32)
    _check(_lib().oracle_aux_scores_bwd_logits(T, E, int(score_fn), _ptr(x), _ptr(g), _ptr(gl)),
           "aux_scores_bwd_logits")
    return gl


def aux_scores_bwd(probs, grad_probs, score_fn: int = 0) -> np.ndarray:
    """dL/dlogits of the softmax aux scores given dL/dprobs (rows of probs sum to 1)."""
    p = np.ascontiguousarray(as_numpy(probs), dtype=np.float32)
    g = np.ascontiguousarray(as_numpy(grad_probs), dtype=np.float32)
    T, E = p.shape
    gl = np.zeros((T, E), np.float32)
    _check(_lib().oracle_aux_scores_bwd(T, E, int(score_fn), _ptr(p), _ptr(g), _ptr(gl)), "aux_scores_bwd")
    return gl


def dispatch(hidden, e2p, p2t, P: int, max_padded: int, fill: int = 0xFFFF) -> np.ndarray:
    """Rows at or past P keep ``fill`` (so tests see that they are untouched)."""
    h = as_numpy(hidden)
    assert h.dtype == np.uint16
    T, H = h.shape
    e2p = np.ascontiguousarray(as_numpy(e2p), dtype=np.int32).ravel()
    k = e2p.size // max(T, 1) if T else 1
    p2t = np.ascontiguousarray(as_numpy(p2t), dtype=np.int32).ravel()
    out = np.full((max_padded, H), fill, np.uint16)
    rc = _lib().oracle_dispatch(T, H, k, _ptr(h), _ptr(e2p), _ptr(p2t), int(P), _ptr(out))
    _check(rc, "dispatch")
    return out


def combine(expert_out, e2p, weights, k: int) -> np.ndarray:
    """Weighted sum of each token's k expert rows: bf16 rows -> bf16 tokens, fp32 rows -> fp32 tokens."""
    eo = as_numpy(expert_out)
    assert eo.dtype in (np.uint16, np.float32)
    w = as_numpy(weights)
    e2p = np.ascontiguousarray(as_numpy(e2p), dtype=np.int32).ravel()
    T = e2p.size // k
    H = eo.shape[1]
    out = np.zeros((T, H), eo.dtype)
    fn = _lib().oracle_combine if eo.dtype == np.uint16 else _lib().oracle_combine_f32
    rc = fn(T, H, k, _ptr(eo), _ptr(e2p), _ptr(np.ascontiguousarray(w)), _dtype_code(w), _ptr(out))
    _check(rc, "combine")
    return out


def rmsnorm_router_topk(hidden, gamma, W, bias, *, k: int, eps: float = 1e-6, act: int = SIGMOID) -> dict:
    x = as_numpy(hidden)
    g = as_numpy(gamma)
    w = as_numpy(W)
    b = as_numpy(bias) if bias is not None else None
    T, H = x.shape
    E = w.shape[1]
    xn = np.zeros((T, H), np.uint16)
    ids = np.zeros((T, k), np.int32)
    aff = np.zeros((T, E), np.uint16)
    lg = np.zeros((T, E), np.float32)
    rc = _lib().oracle_rmsnorm_router_topk(T, H, E, k, float(eps), act, _ptr(x), _ptr(g), _ptr(w), _ptr(b),
                                           _ptr(xn), _ptr(ids), _ptr(aff), _ptr(lg))
    _check(rc, "rmsnorm_router_topk")
    return {"out_norm": xn, "ids": ids, "affinities": aff, "logits": lg}


def router_logits(xn, W, bias=None) -> np.ndarray:
    x = as_numpy(xn)
    w = as_numpy(W)
    b = as_numpy(bias) if bias is not None else None
    T, H = x.shape
    E = w.shape[1]
    out = np.zeros((T, E), np.float32)
    rc = _lib().oracle_router_logits(T, H, E, _ptr(x), _ptr(w), _ptr(b), _ptr(out))
    _check(rc, "router_logits")
    return out


def ep_regroup(counts, recv, tile: int) -> dict:
    """Receive-order rows -> the receiving rank's tile-padded expert layout (expert, source, token)."""
    c = np.ascontiguousarray(as_numpy(counts), dtype=np.int32)
    W, L = c.shape
    r = np.ascontiguousarray(as_numpy(recv))
    n = r.shape[0]
    row_bytes = r.dtype.itemsize * int(np.prod(r.shape[1:]))
    tot = c.sum(0)
    P = int(sum((int(t) + tile - 1) // tile * tile for t in tot))
    padded = np.zeros((max(P, 1),) + r.shape[1:], r.dtype)
    offsets = np.zeros(L + 1, np.int32)
    totals = np.zeros(2, np.int32)
    p2r = np.zeros(max(P, 1), np.int32)
    rc = _lib().oracle_ep_regroup(W, L, tile, _ptr(c), _ptr(r), n, row_bytes, _ptr(padded), _ptr(offsets),
                                  _ptr(totals), _ptr(p2r))
    _check(rc, "ep_regroup")
    return {"padded": padded[:P], "offsets": offsets, "totals": totals, "padded_to_recv": p2r[:P]}
