"""Thin ctypes binding over libmoeroute.so (argument marshalling only).

Every step of the routing path runs in the library's CUDA kernels; this module
only turns torch tensors into device pointers, allocates caller-owned outputs
and workspaces with torch, and checks status codes.  There is no CPU or eager
fallback: if the library is missing or no GPU is present the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoeroute.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_WORKSPACE = -3
MOE_ERR_CUDA = -4
MOE_ERR_DEVICE_TIMEOUT = -5
MOE_ERR_DEVICE_BOUNDS = -6

F32 = 0
BF16 = 1
SOFTMAX = 0
SIGMOID = 1

_DT = {torch.float32: F32, torch.bfloat16: BF16}
_TORCH = {F32: torch.float32, BF16: torch.bfloat16}

# every symbol the C header declares (checked by the CPU test suite)
EXPORTED = (
    "moe_error_string", "moe_workspace_init", "moe_status", "moe_route_capacity",
    "moe_route_workspace_bytes", "moe_route", "moe_aux_workspace_bytes", "moe_aux_scores", "moe_aux_scores_bwd", "moe_aux_scores_bwd_logits", "moe_debug_div_check",
    "moe_route_weights_bwd",
    "moe_aux_loss_fwd", "moe_aux_loss_bwd", "moe_dispatch", "moe_combine",
    "moe_rmsnorm_router_topk_workspace_bytes", "moe_rmsnorm_router_topk", "moe_debug_wait_timeout",
    "moe_debug_sigmoid_proxy_error", "moe_route_no_alloc", "moe_route_no_alloc_status",
    "moe_debug_no_alloc_record", "moe_ep_regroup",
)


class MoeError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {code} ({error_string(code)})")


class RouteParams(ctypes.Structure):
    _fields_ = [
        ("num_tokens", ctypes.c_int32), ("num_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
        ("score_fn", ctypes.c_int32), ("softmax_before_topk", ctypes.c_int32),
        ("n_group", ctypes.c_int32), ("topk_group", ctypes.c_int32), ("group_score_topn", ctypes.c_int32),
        ("renormalize", ctypes.c_int32), ("scaling_factor", ctypes.c_float),
        ("tile_tokens_dim", ctypes.c_int32), ("logits_dtype", ctypes.c_int32), ("bias_dtype", ctypes.c_int32),
        ("weights_dtype", ctypes.c_int32),
        ("local_expert_offset", ctypes.c_int32), ("local_num_experts", ctypes.c_int32),
        ("num_fused_shared_experts", ctypes.c_int32),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load the CUDA library; raise loudly if it was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing (run __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        i32 = ctypes.c_int32
        i64 = ctypes.c_int64
        f32 = ctypes.c_float
        sz = ctypes.c_size_t
        RP = ctypes.POINTER(RouteParams)
        sig = {
            "moe_error_string": ([ctypes.c_int], ctypes.c_char_p),
            "moe_workspace_init": ([P, sz, P], ctypes.c_int),
            "moe_status": ([P, P, ctypes.POINTER(i32), ctypes.c_int], ctypes.c_int),
            "moe_route_capacity": ([RP, ctypes.POINTER(i64), ctypes.POINTER(i64)], ctypes.c_int),
            "moe_route_workspace_bytes": ([RP, ctypes.POINTER(sz)], ctypes.c_int),
            "moe_route": ([RP, P, P, P, P, P, P, P, P, P, P, P, P, sz, P], ctypes.c_int),
            "moe_route_no_alloc": ([RP, P, P, P, P, P, P, P, P, P, P, P, P], ctypes.c_int),
            "moe_route_no_alloc_status": ([P, ctypes.POINTER(i32), ctypes.c_int], ctypes.c_int),
            "moe_debug_no_alloc_record": ([i32, P], ctypes.c_int),
            "moe_ep_regroup": ([i32, i32, i32, i32, i32, P, i32, P, i64, P, i64, P, P, P, P, sz, P], ctypes.c_int),
            "moe_aux_workspace_bytes": ([i32, i32, ctypes.POINTER(sz)], ctypes.c_int),
            "moe_aux_scores": ([i32, i32, i32, i32, P, P, P, P, P, sz, P], ctypes.c_int),
            "moe_aux_loss_fwd": ([i32, i32, i32, i32, f32, P, P, P, P, sz, P], ctypes.c_int),
            "moe_aux_loss_bwd": ([i32, i32, i32, i32, f32, P, P, P, P, P, P], ctypes.c_int),
            "moe_aux_scores_bwd": ([i32, i32, i32, P, P, P, P], ctypes.c_int),
            "moe_aux_scores_bwd_logits": ([i32, i32, i32, P, P, P, P], ctypes.c_int),
            "moe_debug_div_check": ([P, P, ctypes.c_int64, P, P], ctypes.c_int),
            "moe_route_weights_bwd": ([RP, P, P, P, P, P, sz, P], ctypes.c_int),
            "moe_dispatch": ([i32, i32, i32, i32, P, P, P, P, i64, P, P], ctypes.c_int),
            "moe_combine": ([i32, i32, i32, i32, P, i64, P, P, i32, P, P, sz, P], ctypes.c_int),
            "moe_rmsnorm_router_topk_workspace_bytes": ([i32, i32, i32, ctypes.POINTER(sz)], ctypes.c_int),
            "moe_rmsnorm_router_topk": ([i32, i32, i32, i32, f32, i32, P, P, P, P, P, P, P, P, P, sz, P],
                                        ctypes.c_int),
            "moe_debug_wait_timeout": ([i32, i64, P, sz, P], ctypes.c_int),
            "moe_debug_sigmoid_proxy_error": ([P, P, i64, i32, P, P, P], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name, None)
            if fn is None:
                continue
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def error_string(code: int) -> str:
    try:
        return lib().moe_error_string(code).decode()
    except Exception:  # pragma: no cover
        return "?"


def _check(rc: int, what: str):
    if rc != MOE_OK:
        raise MoeError(rc, what)


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def make_workspace(nbytes: int, device) -> torch.Tensor:
    """A zero-filled workspace (what a workspace needs before its first use)."""
    return torch.zeros(max(int(nbytes), 64), dtype=torch.uint8, device=device)


def status(ws: torch.Tensor, clear: bool = True, stream=None) -> int:
    st = ctypes.c_int32(0)
    _check(lib().moe_status(_p(ws), _stream(stream), ctypes.byref(st), int(clear)), "moe_status")
    return int(st.value)


def route_params(T: int, E: int, k: int, *, score_fn: int = SOFTMAX, softmax_before_topk: int = 1,
                 n_group: int = 0, topk_group: int = 0, group_score_topn: int = 2, renormalize: int = 1,
                 scaling_factor: float = 1.0, tile_tokens_dim: int = 8, logits_dtype: int = F32,
                 bias_dtype: int = F32, weights_dtype: int = F32, local_expert_offset: int = 0,
                 local_num_experts: int = 0, num_fused_shared_experts: int = 0) -> RouteParams:
    """local_num_experts == 0: every expert is local (single GPU)."""
    return RouteParams(T, E, k, score_fn, softmax_before_topk, n_group, topk_group, group_score_topn,
                       renormalize, scaling_factor, tile_tokens_dim, logits_dtype, bias_dtype, weights_dtype,
                       local_expert_offset, local_num_experts, num_fused_shared_experts)


def route_capacity(p: RouteParams):
    mp, mt = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().moe_route_capacity(ctypes.byref(p), ctypes.byref(mp), ctypes.byref(mt)), "moe_route_capacity")
    return int(mp.value), int(mt.value)


class Router:
    """Caller-owned outputs + workspace for repeated moe_route calls of one shape."""

    def __init__(self, p: RouteParams, device="cuda"):
        self.p = p
        self.device = torch.device(device)
        L = lib()
        self.max_padded, self.max_tiles = route_capacity(p)
        nb = ctypes.c_size_t()
        with torch.cuda.device(self.device):
            _check(L.moe_route_workspace_bytes(ctypes.byref(p), ctypes.byref(nb)), "moe_route_workspace_bytes")
        dev = self.device
        T, E, S = p.num_tokens, p.num_experts, p.num_fused_shared_experts
        k = p.top_k + S  # slots per token: the routed ones, then the fused shared ones
        L_e = (p.local_num_experts if p.local_num_experts > 0 else E) + S  # the local experts' bookkeeping
        self.ws = make_workspace(nb.value, dev)
        self.out = {
            "ids": torch.empty((T, k), dtype=torch.int32, device=dev),
            "weights": torch.empty((T, k), dtype=_TORCH[p.weights_dtype], device=dev),
            "counts": torch.empty(L_e, dtype=torch.int32, device=dev),
            "offsets": torch.empty(L_e + 1, dtype=torch.int32, device=dev),
            "e2p": torch.empty(T * k, dtype=torch.int32, device=dev),
            "p2t": torch.empty(max(self.max_padded, 1), dtype=torch.int32, device=dev),
            "tile_expert": torch.empty(max(self.max_tiles, 1), dtype=torch.int32, device=dev),
            "tile_mn_limit": torch.empty(max(self.max_tiles, 1), dtype=torch.int32, device=dev),
            "totals": torch.empty(2, dtype=torch.int32, device=dev),
        }
        o = self.out
        self._ptrs = [_p(o[n]) for n in ("ids", "weights", "counts", "offsets", "e2p", "p2t", "tile_expert",
                                         "tile_mn_limit", "totals")]
        self._ws = (_p(self.ws), ctypes.c_size_t(self.ws.numel()))

    def __call__(self, logits: torch.Tensor, bias: Optional[torch.Tensor] = None, stream=None) -> Dict[str, torch.Tensor]:
        p = self.p
        if logits.dtype != _TORCH[p.logits_dtype] or tuple(logits.shape) != (p.num_tokens, p.num_experts):
            raise ValueError("logits shape/dtype do not match the router parameters")
        if bias is not None and (bias.dtype != _TORCH[p.bias_dtype] or bias.numel() != p.num_experts):
            raise ValueError("bias shape/dtype do not match the router parameters")
        rc = lib().moe_route(ctypes.byref(p), _p(logits), _p(bias), *self._ptrs, *self._ws, _stream(stream))
        _check(rc, "moe_route")
        return self.out


def route(logits: torch.Tensor, bias: Optional[torch.Tensor] = None, *, k: int, **kw) -> Dict[str, torch.Tensor]:
    """One-shot moe_route with freshly allocated outputs (see Router for repeated calls)."""
    T, E = logits.shape
    p = route_params(T, E, k, logits_dtype=_DT[logits.dtype],
                     bias_dtype=_DT[bias.dtype] if bias is not None else F32, **kw)
    r = Router(p, logits.device)
    out = dict(r(logits, bias))
    out["ws"] = r.ws
    out["max_padded"] = r.max_padded
    out["max_tiles"] = r.max_tiles
    return out


def debug_wait_timeout(never_complete: bool, timeout_ns: int, ws: torch.Tensor, stream=None):
    _check(lib().moe_debug_wait_timeout(int(never_complete), timeout_ns, _p(ws), ctypes.c_size_t(ws.numel()),
                                        _stream(stream)), "moe_debug_wait_timeout")


def route_into(p: RouteParams, logits: torch.Tensor, bias: Optional[torch.Tensor], out: Dict[str, torch.Tensor],
               ws: torch.Tensor, stream=None) -> None:
    """moe_route into caller-provided output tensors (names as in Router.out)."""
    names = ("ids", "weights", "counts", "offsets", "e2p", "p2t", "tile_expert", "tile_mn_limit", "totals")
    rc = lib().moe_route(ctypes.byref(p), _p(logits), _p(bias), *[_p(out[n]) for n in names], _p(ws),
                         ctypes.c_size_t(ws.numel()), _stream(stream))
    _check(rc, "moe_route")


def route_weights_bwd_into(p: RouteParams, logits: torch.Tensor, ids: torch.Tensor, grad_weights: torch.Tensor,
                           grad_logits: torch.Tensor, ws: Optional[torch.Tensor] = None, stream=None) -> None:
    _check(lib().moe_route_weights_bwd(ctypes.byref(p), _p(logits), _p(ids), _p(grad_weights), _p(grad_logits),
                                       _p(ws), ctypes.c_size_t(ws.numel() if ws is not None else 0),
                                       _stream(stream)),
           "moe_route_weights_bwd")


def route_weights_bwd(p: RouteParams, logits: torch.Tensor, ids: torch.Tensor, grad_weights: torch.Tensor,
                      ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """moe_route_weights_bwd: dL/dlogits [T,E] fp32 from dL/dweights [T,k] fp32 for the given selection."""
    T, E = logits.shape
    gl = torch.empty((T, E), dtype=torch.float32, device=logits.device)
    route_weights_bwd_into(p, logits, ids, grad_weights, gl, ws, stream)
    return gl


def route_workspace_bytes(p: RouteParams) -> int:
    nb = ctypes.c_size_t()
    _check(lib().moe_route_workspace_bytes(ctypes.byref(p), ctypes.byref(nb)), "moe_route_workspace_bytes")
    return int(nb.value)


def debug_sigmoid_proxy_error(x: torch.Tensor, b: torch.Tensor, f32_logits: bool = False, stream=None):
    """(proxy - exact key, the assumed bound) per element, for logits x and biases b (fp32 device tensors)."""
    err = torch.empty_like(x)
    delta = torch.empty_like(x)
    _check(lib().moe_debug_sigmoid_proxy_error(_p(x), _p(b), x.numel(), int(f32_logits), _p(err), _p(delta),
                                               _stream(stream)), "moe_debug_sigmoid_proxy_error")
    return err, delta


# ---------------------------------------------------------------------------- aux loss

def aux_workspace(T: int, E: int, device) -> torch.Tensor:
    nb = ctypes.c_size_t()
    _check(lib().moe_aux_workspace_bytes(T, E, ctypes.byref(nb)), "moe_aux_workspace_bytes")
    return make_workspace(nb.value, device)


def aux_scores_into(logits: torch.Tensor, k: int, probs: torch.Tensor, routing_map: torch.Tensor,
                    tokens_per_expert: torch.Tensor, ws: torch.Tensor, score_fn: int = SOFTMAX, stream=None) -> None:
    T, E = logits.shape
    _check(lib().moe_aux_scores(T, E, k, score_fn, _p(logits), _p(probs), _p(routing_map), _p(tokens_per_expert),
                                _p(ws), ctypes.c_size_t(ws.numel()), _stream(stream)), "moe_aux_scores")


def aux_scores(logits: torch.Tensor, k: int, score_fn: int = SOFTMAX, ws: Optional[torch.Tensor] = None):
    T, E = logits.shape
    dev = logits.device
    probs = torch.empty((T, E), dtype=torch.float32, device=dev)
    rmap = torch.empty((T, E), dtype=torch.uint8, device=dev)
    tpe = torch.empty(E, dtype=torch.int32, device=dev)
    ws = aux_workspace(T, E, dev) if ws is None else ws
    aux_scores_into(logits, k, probs, rmap, tpe, ws, score_fn)
    return {"probs": probs, "routing_map": rmap, "tokens_per_expert": tpe, "ws": ws}


def aux_loss_fwd_into(probs: torch.Tensor, tokens_per_expert: torch.Tensor, T_total: int, k: int, coeff: float,
                      loss: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    T, E = probs.shape
    _check(lib().moe_aux_loss_fwd(T, T_total, E, k, coeff, _p(probs), _p(tokens_per_expert), _p(loss), _p(ws),
                                  ctypes.c_size_t(ws.numel()), _stream(stream)), "moe_aux_loss_fwd")


def aux_loss_fwd(probs: torch.Tensor, tokens_per_expert: torch.Tensor, T_total: int, k: int, coeff: float,
                 ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    T, E = probs.shape
    loss = torch.empty(1, dtype=torch.float32, device=probs.device)
    ws = aux_workspace(T, E, probs.device) if ws is None else ws
    aux_loss_fwd_into(probs, tokens_per_expert, T_total, k, coeff, loss, ws)
    return loss


def aux_loss_bwd_into(grad_loss: torch.Tensor, probs: torch.Tensor, tokens_per_expert: torch.Tensor, T_total: int,
                      k: int, coeff: float, grad_probs: Optional[torch.Tensor], grad_logits: Optional[torch.Tensor],
                      stream=None) -> None:
    T, E = probs.shape
    _check(lib().moe_aux_loss_bwd(T, T_total, E, k, coeff, _p(grad_loss), _p(probs), _p(tokens_per_expert),
                                  _p(grad_probs), _p(grad_logits), _stream(stream)), "moe_aux_loss_bwd")


def aux_loss_bwd(grad_loss: torch.Tensor, probs: torch.Tensor, tokens_per_expert: torch.Tensor, T_total: int, k: int,
                 coeff: float, want_grad_probs: bool = True):
    gp = torch.empty_like(probs) if want_grad_probs else None
    gl = torch.empty_like(probs)
    aux_loss_bwd_into(grad_loss, probs, tokens_per_expert, T_total, k, coeff, gp, gl)
    return {"grad_probs": gp, "grad_logits": gl}


def aux_scores_bwd_into(probs: torch.Tensor, grad_probs: torch.Tensor, grad_logits: torch.Tensor,
                        score_fn: int = SOFTMAX, stream=None) -> None:
    T, E = probs.shape
    _check(lib().moe_aux_scores_bwd(T, E, score_fn, _p(probs), _p(grad_probs), _p(grad_logits), _stream(stream)),
           "moe_aux_scores_bwd")


def aux_scores_bwd_logits_into(logits: torch.Tensor, grad_probs: torch.Tensor, grad_logits: torch.Tensor,
                               score_fn: int = SOFTMAX, stream=None) -> None:
    T, E = logits.shape
    _check(lib().moe_aux_scores_bwd_logits(T, E, score_fn, _p(logits), _p(grad_probs), _p(grad_logits),
                                           _stream(stream)), "moe_aux_scores_bwd_logits")


def aux_scores_bwd_logits(logits: torch.Tensor, grad_probs: torch.Tensor, score_fn: int = SOFTMAX) -> torch.Tensor:
    gl = torch.empty_like(logits)
    aux_scores_bwd_logits_into(logits, grad_probs, gl, score_fn)
    return gl


def debug_div_check(a: torch.Tensor, b: torch.Tensor) -> int:
    """Pairs (in the method's range) where the reciprocal-and-corrections quotient differs from a / b."""
    bad = torch.zeros(1, dtype=torch.int32, device=a.device)
    _check(lib().moe_debug_div_check(_p(a), _p(b), a.numel(), _p(bad), _stream(None)), "moe_debug_div_check")
    return int(bad.item())


def aux_scores_bwd(probs: torch.Tensor, grad_probs: torch.Tensor, score_fn: int = SOFTMAX) -> torch.Tensor:
    """dL/dlogits of the aux scores given dL/dprobs."""
    gl = torch.empty_like(probs)
    aux_scores_bwd_into(probs, grad_probs, gl, score_fn)
    return gl


# ---------------------------------------------------------------------------- dispatch / combine

def dispatch_into(hidden: torch.Tensor, e2p: torch.Tensor, p2t: torch.Tensor, totals: torch.Tensor, k: int,
                  out: torch.Tensor, stream=None) -> None:
    T, H = hidden.shape
    _check(lib().moe_dispatch(T, H, k, _DT[hidden.dtype], _p(hidden), _p(e2p), _p(p2t), _p(totals), out.shape[0],
                              _p(out), _stream(stream)), "moe_dispatch")


def combine_into(expert_out: torch.Tensor, e2p: torch.Tensor, weights: torch.Tensor, k: int, out: torch.Tensor,
                 ws: Optional[torch.Tensor] = None, stream=None) -> None:
    T, H = out.shape
    _check(lib().moe_combine(T, H, k, _DT[expert_out.dtype], _p(expert_out), expert_out.shape[0], _p(e2p),
                             _p(weights), _DT[weights.dtype], _p(out), _p(ws),
                             ctypes.c_size_t(0 if ws is None else ws.numel()), _stream(stream)), "moe_combine")


# ---------------------------------------------------------------------------- decode fused

def decode_workspace(T: int, H: int, E: int, device) -> torch.Tensor:
    nb = ctypes.c_size_t()
    _check(lib().moe_rmsnorm_router_topk_workspace_bytes(T, H, E, ctypes.byref(nb)),
           "moe_rmsnorm_router_topk_workspace_bytes")
    return make_workspace(nb.value, device)


def rmsnorm_router_topk_into(hidden, gamma, W, bias, k: int, eps: float, act: int, out_norm, ids, affinities,
                             debug_logits, ws, stream=None) -> None:
    T, H = hidden.shape
    E = W.shape[1]
    _check(lib().moe_rmsnorm_router_topk(T, H, E, k, eps, act, _p(hidden), _p(gamma), _p(W), _p(bias), _p(out_norm),
                                         _p(ids), _p(affinities), _p(debug_logits), _p(ws),
                                         ctypes.c_size_t(ws.numel()), _stream(stream)), "moe_rmsnorm_router_topk")


def rmsnorm_router_topk(hidden, gamma, W, bias=None, *, k: int, eps: float = 1e-6, act: int = SIGMOID,
                        debug_logits: bool = False, ws: Optional[torch.Tensor] = None):
    T, H = hidden.shape
    E = W.shape[1]
    dev = hidden.device
    out_norm = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    aff = torch.empty((T, E), dtype=torch.bfloat16, device=dev)
    lg = torch.empty((T, E), dtype=torch.float32, device=dev) if debug_logits else None
    ws = decode_workspace(T, H, E, dev) if ws is None else ws
    rmsnorm_router_topk_into(hidden, gamma, W, bias, k, eps, act, out_norm, ids, aff, lg, ws)
    return {"out_norm": out_norm, "ids": ids, "affinities": aff, "logits": lg, "ws": ws}


def route_no_alloc_into(p: RouteParams, logits: torch.Tensor, bias: Optional[torch.Tensor],
                        out: Dict[str, torch.Tensor], stream=None) -> None:
    """moe_route_no_alloc: like route_into, with the library's own static workspace (no allocation)."""
    names = ("ids", "weights", "counts", "offsets", "e2p", "p2t", "tile_expert", "tile_mn_limit", "totals")
    rc = lib().moe_route_no_alloc(ctypes.byref(p), _p(logits), _p(bias), *[_p(out[n]) for n in names],
                                  _stream(stream))
    _check(rc, "moe_route_no_alloc")


def route_no_alloc_status(clear: bool = True, stream=None) -> int:
    """The status word of moe_route_no_alloc's static workspace (sticky until cleared)."""
    st = ctypes.c_int32(0)
    _check(lib().moe_route_no_alloc_status(_stream(stream), ctypes.byref(st), int(clear)), "moe_route_no_alloc_status")
    return int(st.value)


# ---------------------------------------------------------------------------- expert-parallel exchange

def ep_regroup_into(counts: torch.Tensor, recv: torch.Tensor, padded: torch.Tensor, tile: int, offsets: torch.Tensor,
                    totals: torch.Tensor, padded_to_recv: torch.Tensor, ws: Optional[torch.Tensor] = None,
                    stream=None) -> None:
    """Receive order -> tile-padded expert layout (moe_ep_regroup, direction 0)."""
    W, L = counts.shape
    H = recv.shape[1]
    _check(lib().moe_ep_regroup(W, L, H, _DT[recv.dtype], tile, _p(counts), 0, _p(recv), recv.shape[0], _p(padded),
                                padded.shape[0], _p(offsets), _p(totals), _p(padded_to_recv), _p(ws),
                                ctypes.c_size_t(0 if ws is None else ws.numel()), _stream(stream)), "moe_ep_regroup")


def ep_ungroup_into(counts: torch.Tensor, padded: torch.Tensor, recv: torch.Tensor, tile: int,
                    ws: Optional[torch.Tensor] = None, stream=None) -> None:
    """Tile-padded expert layout -> receive order (moe_ep_regroup, direction 1)."""
    W, L = counts.shape
    H = recv.shape[1]
    _check(lib().moe_ep_regroup(W, L, H, _DT[recv.dtype], tile, _p(counts), 1, _p(recv), recv.shape[0], _p(padded),
                                padded.shape[0], None, None, None, _p(ws),
                                ctypes.c_size_t(0 if ws is None else ws.numel()), _stream(stream)), "moe_ep_regroup")
