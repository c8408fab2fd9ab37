"""Expert-parallel dispatch and combine over a real process group: gloo ranks on the CPU, the per-rank
steps by the oracle (stand-ins for the CUDA library), the collectives and the exchange logic as
top_expert_selection_b200.ep runs them.  Each rank's expert input must equal the single-process shard
route of all ranks' tokens concatenated in rank order, and each rank's combined rows the combine of its
own tokens."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import numpy as np
    import torch.distributed as dist

    import ep_common as C
    import oracle
    from top_expert_selection_b200.ep import EpExchange, TorchComm

    class GlooComm(TorchComm):
        # gloo moves raw bytes: bf16 rows travel as bytes
        def all_to_all(self, o, i, os_=None, is_=None):
            if o.dtype == torch.bfloat16:
                o, i = o.view(torch.uint8), i.view(torch.uint8)
            super().all_to_all(o, i, os_, is_)

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        lg, hidden = C.rank_inputs(rank)
        sel, route = C.oracle_route(lg)
        ep = EpExchange(world, rank, C.E, C.K, C.TILE, comm=GlooComm(), ops=C.OracleOps())
        padded, st = ep.dispatch(hidden, route)
        ref, ref_bk = C.reference_expert_input(rank, world)
        P = int(st.totals[0])
        ok_in = (P == int(ref_bk["totals"][0]) and st.offsets.tolist() == ref_bk["offsets"].tolist()
                 and np.array_equal(oracle.as_numpy(padded[:P]), ref))
        res = ep.combine(C.expert_fn(padded[:P]), st, sel["weights"], hidden.shape[0])
        rows = C.OracleOps().dispatch(hidden, route, C.K, hidden.shape[0] * C.K)
        own = C.OracleOps().combine(C.expert_fn(rows), route, sel["weights"], C.K, hidden.shape[0])
        ok_out = torch.equal(res.view(torch.int16), own.view(torch.int16))
        out.put((rank, ok_in, ok_out, P))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ep_exchange_over_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok_in, ok_out, P in sorted(res):
        assert ok_in, f"rank {rank}: expert input differs from the single-process shard route"
        assert ok_out, f"rank {rank}: combined rows differ from its own tokens' combine"
