"""Host logic of the multi-GPU bench path on CPU: two gloo ranks (no GPU).

bench.py runs one process per GPU; each rank routes its own seeded batch of the
same shape (weak scaling, no collective on the data path) and the timed
milliseconds are reduced with a max over ranks before the whole-job rate is
formed.  These ranks exercise exactly those helpers over a real process group.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, dist, "cpu")
        spec = bench.rank_spec(rank)
        rate = bench.whole_job_rate(world, spec.T, ms)
        dist.barrier()
        out.put((rank, ms, rate, spec.seed, spec.T))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    (r0, ms0, rate0, seed0, T0), (r1, ms1, rate1, seed1, T1) = res
    assert ms0 == ms1 == 15.0, "timing must be the max over ranks on every rank"
    assert rate0 == rate1 == pytest.approx(2 * T0 / 0.015)
    assert T0 == T1 and seed0 != seed1, "same shape, different seeded batch per rank"


def test_single_process_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
    assert bench.whole_job_rate(1, 16384, 0.5) == pytest.approx(16384 / 0.0005)
