"""Expert-parallel dispatch and combine over an all-to-all-v (one process per GPU).

The router's top-k feeds the all-to-all-v MoE dispatch path (RMSNorm Router
Top-K A2AV Kernel API Reference, Background); a rank owns a contiguous range of
experts (flashinfer.fused_moe.trtllm_gen_routing, Parameters local_expert_offset
/ local_num_experts).

World of W ranks, E experts, L = E / W per rank.  Every rank routes its own
tokens over all E experts with tile 1 (moe_route), so its dispatched rows
(moe_dispatch) are ordered by expert, then token: the rows for destination d
are one contiguous run (experts d*L .. d*L+L-1).  Then:

  1. counts: an all-to-all of the per-expert counts (L ints to every rank);
  2. rows: an all-to-all-v of the dispatched rows (row splits from the counts);
  3. moe_ep_regroup lays the received rows out by local expert, then source
     rank, then token, tile-padded: the grouped GEMM's input, identical to the
     layout one route of all ranks' tokens (concatenated in rank order) gives
     this rank's experts;
  4. the return: moe_ep_regroup (direction 1) puts the expert outputs back in
     receive order, the reverse all-to-all-v sends them home, and moe_combine
     forms each token's weighted sum in its tile-1 layout.

Remote rows always land in local buffers (NCCL copies); no kernel reads a
peer's memory.  The collectives go through `comm` (torch.distributed by
default) and the per-rank steps through `ops` (the CUDA library by default);
the split sizes are read back to the host once per exchange.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import torch


class TorchComm:
    """The all-to-alls through torch.distributed (NCCL for CUDA tensors)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group

    def all_to_all(self, out: torch.Tensor, inp: torch.Tensor, out_splits: Optional[List[int]] = None,
                   in_splits: Optional[List[int]] = None) -> None:
        self.dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)


class CudaOps:
    """The per-rank steps on the GPU (libmoeroute)."""

    def __init__(self):
        from . import binding as B
        self.B = B

    def dispatch(self, hidden, route, k, max_rows):
        out = torch.empty((max(max_rows, 1), hidden.shape[1]), dtype=hidden.dtype, device=hidden.device)
        self.B.dispatch_into(hidden, route["e2p"], route["p2t"], route["totals"], k, out)
        return out[:max_rows]

    def regroup(self, counts, recv, tile, max_padded):
        dev = recv.device
        H = recv.shape[1]
        padded = torch.empty((max(max_padded, 1), H), dtype=recv.dtype, device=dev)
        L = counts.shape[1]
        offsets = torch.empty(L + 1, dtype=torch.int32, device=dev)
        totals = torch.empty(2, dtype=torch.int32, device=dev)
        p2r = torch.empty(max(max_padded, 1), dtype=torch.int32, device=dev)
        self.B.ep_regroup_into(counts, recv, padded, tile, offsets, totals, p2r)
        return {"padded": padded, "offsets": offsets, "totals": totals, "padded_to_recv": p2r}

    def ungroup(self, counts, padded, n_recv, tile):
        recv = torch.empty((max(n_recv, 1), padded.shape[1]), dtype=padded.dtype, device=padded.device)
        self.B.ep_ungroup_into(counts, padded, recv[:n_recv], tile)
        return recv[:n_recv]

    def combine(self, rows, route, weights, k, T):
        out = torch.empty((T, rows.shape[1]), dtype=rows.dtype, device=rows.device)
        if T:
            self.B.combine_into(rows, route["e2p"], weights, k, out)
        return out


@dataclass
class EpState:
    """What the return path needs from the dispatch."""
    send_counts: torch.Tensor  # [W, L] rows this rank sent per destination and expert
    recv_counts: torch.Tensor  # [W, L] rows this rank received per source and local expert
    send_splits: List[int]
    recv_splits: List[int]
    route: dict                # this rank's tile-1 route over all experts
    offsets: torch.Tensor      # [L + 1] padded offsets of the local experts
    totals: torch.Tensor       # [2] P, P / tile
    padded_to_recv: torch.Tensor


class EpExchange:
    """One rank's side of the expert-parallel exchange."""

    def __init__(self, world: int, rank: int, num_experts: int, top_k: int, tile: int, comm=None, ops=None):
        if num_experts % world != 0:
            raise ValueError("experts must split evenly over the ranks")
        self.W, self.rank, self.E, self.k, self.tile = world, rank, num_experts, top_k, tile
        self.L = num_experts // world
        self.comm = comm if comm is not None else TorchComm()
        self.ops = ops if ops is not None else CudaOps()

    # -- steps (each rank runs them in the same order; the collectives pair up) --
    def send_counts(self, route) -> torch.Tensor:
        """[W, L]: rows for destination d's local expert e (the route's counts, tile 1, all experts)."""
        return route["counts"].reshape(self.W, self.L).to(torch.int32).contiguous()

    def exchange_counts(self, send_counts: torch.Tensor) -> torch.Tensor:
        recv = torch.empty_like(send_counts)
        self.comm.all_to_all(recv.view(-1), send_counts.view(-1))
        return recv

    def dispatch(self, hidden: torch.Tensor, route: dict):
        """hidden [T, H] and this rank's route (tile 1, all experts) -> (padded expert input, state)."""
        T = hidden.shape[0]
        sc = self.send_counts(route)
        rc = self.exchange_counts(sc)
        send_splits = [int(v) for v in sc.sum(1).tolist()]
        recv_splits = [int(v) for v in rc.sum(1).tolist()]
        send = self.ops.dispatch(hidden, route, self.k, T * self.k)
        n_recv = sum(recv_splits)
        recv = torch.empty((n_recv, hidden.shape[1]), dtype=hidden.dtype, device=hidden.device)
        self.comm.all_to_all(recv, send, recv_splits, send_splits)
        max_padded = n_recv + self.L * (self.tile - 1)
        g = self.ops.regroup(rc, recv, self.tile, max_padded)
        st = EpState(sc, rc, send_splits, recv_splits, route, g["offsets"], g["totals"], g["padded_to_recv"])
        return g["padded"], st

    def combine(self, expert_out: torch.Tensor, st: EpState, weights: torch.Tensor, T: int) -> torch.Tensor:
        """Expert outputs in the padded layout -> this rank's tokens [T, H] (weighted sums)."""
        n_recv = sum(st.recv_splits)
        back = self.ops.ungroup(st.recv_counts, expert_out, n_recv, self.tile)
        home = torch.empty((T * self.k, expert_out.shape[1]), dtype=expert_out.dtype, device=expert_out.device)
        self.comm.all_to_all(home, back, st.send_splits, st.recv_splits)
        return self.ops.combine(home, st.route, weights, self.k, T)
