"""The expert-parallel exchange with the CUDA library on one GPU: W ranks as threads of one process, the
all-to-alls done in process (copies between the ranks' device buffers), every per-rank step --
moe_route (tile 1, all experts), moe_dispatch, moe_ep_regroup in both directions, moe_combine -- on the
GPU.  Each rank's expert input must equal the oracle's single-process shard route of all ranks' tokens
concatenated in rank order (bit-exact copy), and each rank's combined rows the oracle's combine of its
own tokens with the same weights (bit-exact: both accumulate in slot order in fp32)."""
import threading

import numpy as np
import pytest
import torch

import ep_common as C
import oracle
from parity import to_np
from top_expert_selection_b200 import binding as B
from top_expert_selection_b200 import workloads as W
from top_expert_selection_b200.ep import CudaOps, EpExchange

pytestmark = pytest.mark.gpu


def _gpu_route(logits):
    T = logits.shape[0]
    p = B.route_params(T, C.E, C.K, score_fn=W.SOFTMAX, softmax_before_topk=0, renormalize=0, tile_tokens_dim=1,
                       logits_dtype=W.BF16, weights_dtype=W.F32)
    r = B.Router(p)
    return r(logits.cuda()) if T else r(torch.empty((0, C.E), dtype=torch.bfloat16, device="cuda"))


@pytest.mark.parametrize("world", [2, 4])
def test_ep_exchange_cuda_in_process(world):
    shared = C.make_shared(world)
    results = [None] * world
    errors = []

    def run(rank):
        try:
            lg, hidden = C.rank_inputs(rank)
            route = _gpu_route(lg)
            hid = hidden.cuda()
            ep = EpExchange(world, rank, C.E, C.K, C.TILE, comm=C.ThreadComm(rank, shared), ops=CudaOps())
            padded, st = ep.dispatch(hid, route)
            torch.cuda.synchronize()
            P = int(st.totals[0])
            out = ep.combine(C.expert_fn(padded[:P]), st, route["weights"], hid.shape[0])
            torch.cuda.synchronize()
            results[rank] = (to_np(route["ids"]), to_np(route["weights"]), to_np(padded[:P]), to_np(st.offsets),
                             int(st.totals[0]), to_np(out), to_np(st.padded_to_recv[:P]))
        except Exception as exc:  # reported by the main thread
            errors.append((rank, exc))
            shared["barrier"].abort()

    threads = [threading.Thread(target=run, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not errors, errors
    for rank in range(world):
        ids, w, padded, offsets, P, out, p2r = results[rank]
        sel, _ = C.oracle_route(C.rank_inputs(rank)[0])
        assert np.array_equal(ids, sel["ids"]), "top-2 on bf16 logits has no rounding: ids must agree"
        ref, ref_bk = C.reference_expert_input(rank, world)
        assert P == int(ref_bk["totals"][0]) and offsets.tolist() == ref_bk["offsets"].tolist()
        assert np.array_equal(padded, ref), f"rank {rank}: expert input differs from the oracle"
        assert np.array_equal(p2r >= 0, ref_bk["p2t"][:P] >= 0)
        # the combine of the rank's own tokens (the oracle, the GPU's weights)
        _, hidden = C.rank_inputs(rank)
        bk = oracle.route_bookkeeping(ids, C.E, 1)
        Pt = int(bk["totals"][0])
        rows = oracle.dispatch(hidden, bk["e2p"], bk["p2t"], Pt, max(Pt, 1))[:Pt]
        doubled = oracle.as_numpy(C.expert_fn(C.bf16(rows)))
        own = oracle.combine(doubled, bk["e2p"], w, C.K) if hidden.shape[0] else np.zeros((0, C.H), np.uint16)
        assert np.array_equal(out, own), f"rank {rank}: combined rows differ from the oracle"


def test_ep_regroup_reports_mismatched_counts():
    # counts that promise more rows than the receive buffer holds: nothing moves, the status says so
    counts = torch.tensor([[3, 1], [2, 2]], dtype=torch.int32, device="cuda")
    recv = torch.randn(5, 8, device="cuda")
    padded = torch.full((16, 8), 7.0, device="cuda")
    off = torch.zeros(3, dtype=torch.int32, device="cuda")
    tot = torch.zeros(2, dtype=torch.int32, device="cuda")
    p2r = torch.zeros(16, dtype=torch.int32, device="cuda")
    ws = B.make_workspace(64, "cuda")
    B.ep_regroup_into(counts, recv, padded, 4, off, tot, p2r, ws=ws)
    torch.cuda.synchronize()
    assert B.status(ws) == B.MOE_ERR_DEVICE_BOUNDS
    assert torch.all(padded == 7.0)
