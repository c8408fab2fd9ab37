"""Shared pieces of the expert-parallel exchange tests: seeded per-rank inputs, an in-process
all-to-all between threads, and CPU stand-ins (the oracle) for the per-rank CUDA steps."""
from __future__ import annotations

import threading

import numpy as np
import torch

import oracle
from top_expert_selection_b200 import workloads as W

E, K, H, TILE = 8, 2, 64, 4
TOKENS = (37, 50, 0, 21)  # per rank (rank 2 routes nothing)


def rank_inputs(rank: int):
    """Seeded logits (bf16 N(0,1)) and hidden rows (bf16 N(0,1)) of one rank's tokens."""
    g = torch.Generator().manual_seed(1000 + rank)
    T = TOKENS[rank]
    logits = torch.randn(T, E, generator=g).to(torch.bfloat16)
    hidden = torch.randn(T, H, generator=g).to(torch.bfloat16)
    return logits, hidden


def oracle_route(logits):
    """The rank's route over all experts with tile 1 (top-2 on logits, softmax over the two; fp32 weights)."""
    sel = oracle.route_select(logits, k=K, score_fn=W.SOFTMAX, softmax_before_topk=0, renormalize=0)
    bk = oracle.route_bookkeeping(sel["ids"], E, 1)
    P = int(bk["totals"][0])
    p2t = np.full(max(P, 1), -1, np.int32)
    p2t[:P] = bk["p2t"]
    return sel, {"counts": torch.from_numpy(bk["counts"]), "e2p": torch.from_numpy(bk["e2p"]),
                 "p2t": torch.from_numpy(p2t), "totals": torch.from_numpy(bk["totals"]),
                 "offsets": torch.from_numpy(bk["offsets"])}


def bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


class OracleOps:
    """The per-rank steps on the CPU through the oracle (test stand-ins for the CUDA library)."""

    def dispatch(self, hidden, route, k, max_rows):
        P = int(route["totals"][0])
        out = oracle.dispatch(hidden, route["e2p"].numpy(), route["p2t"].numpy()[:P], P, max(P, 1))
        return bf16(out[:P])

    def regroup(self, counts, recv, tile, max_padded):
        g = oracle.ep_regroup(counts.numpy(), oracle.as_numpy(recv), tile)
        return {"padded": bf16(g["padded"]), "offsets": torch.from_numpy(g["offsets"]),
                "totals": torch.from_numpy(g["totals"]), "padded_to_recv": torch.from_numpy(g["padded_to_recv"])}

    def ungroup(self, counts, padded, n_recv, tile):
        # the inverse of regroup: receive row r comes from the padded row that regroup filled with it
        idx = oracle.ep_regroup(counts.numpy(), np.arange(n_recv, dtype=np.int32).reshape(n_recv, 1), tile)
        out = torch.empty((n_recv, padded.shape[1]), dtype=padded.dtype)
        p2r = idx["padded_to_recv"]
        for p in range(p2r.shape[0]):
            if p2r[p] >= 0:
                out[p2r[p]] = padded[p]
        return out

    def combine(self, rows, route, weights, k, T):
        if T == 0:
            return torch.empty((0, rows.shape[1]), dtype=rows.dtype)
        return bf16(oracle.combine(rows, route["e2p"].numpy(), weights, k))


class ThreadComm:
    """all_to_all_single between threads of one process (one object per rank, a shared exchange)."""

    def __init__(self, rank: int, shared: dict):
        self.rank = rank
        self.shared = shared

    def all_to_all(self, out, inp, out_splits=None, in_splits=None):
        W = self.shared["world"]
        bar = self.shared["barrier"]
        n = inp.shape[0]
        if in_splits is None:
            in_splits = [n // W] * W
        self.shared["inputs"][self.rank] = (inp, in_splits)
        bar.wait()
        pieces = []
        for s in range(W):
            src, splits = self.shared["inputs"][s]
            start = sum(splits[:self.rank])
            pieces.append(src[start:start + splits[self.rank]])
        if pieces:
            res = torch.cat(pieces)
            if res.numel():
                out.copy_(res.to(out.device))
        bar.wait()


def make_shared(world: int) -> dict:
    return {"world": world, "barrier": threading.Barrier(world), "inputs": [None] * world}


def reference_expert_input(rank: int, world: int):
    """The single-process shard route of all ranks' tokens concatenated in rank order, dispatched:
    what rank `rank`'s grouped GEMM must receive."""
    L = E // world
    ids, hid = [], []
    for s in range(world):
        lg, h = rank_inputs(s)
        sel, _ = oracle_route(lg)
        ids.append(sel["ids"])
        hid.append(oracle.as_numpy(h))
    ids = np.concatenate(ids) if ids else np.zeros((0, K), np.int32)
    hid = np.concatenate(hid)
    bk = oracle.route_bookkeeping(ids, E, TILE, rank * L, L)
    P = int(bk["totals"][0])
    ref = oracle.dispatch(hid, bk["e2p"], bk["p2t"], P, max(P, 1))
    return ref[:P], bk


def expert_fn(padded: torch.Tensor) -> torch.Tensor:
    """A stand-in expert: every row doubled (exact in bf16)."""
    return (padded.float() * 2.0).to(padded.dtype)
