"""The multi-rank host logic of bench.py on CPU: two gloo ranks.

Each rank runs an independent layer (its own seeded inputs, weak scaling);
the only collectives are the barrier and the max-over-ranks time reduction,
and the reported value counts every rank's forwards.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        total = bench.max_over_ranks(local_ms, world, "cpu")
        dist.barrier()
        q.put((rank, total, bench.whole_job_value(world, 4, total), bench.rank_seed(rank)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_and_value():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    totals = {r[1] for r in res}
    assert totals == {15.0}                       # max over ranks, seen by every rank
    assert res[0][2] == pytest.approx(2 * 4 / 0.015)
    assert res[0][3] != res[1][3]                 # independent inputs per rank


def test_single_rank_helpers():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.whole_job_value(1, 10, 100.0) == pytest.approx(100.0)
    assert bench.rank_seed(0) == 1002
