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


def _heads_rank_main(rank, world, port, n_heads, q):
    import sys
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from free_clustered_block_b200 import heads, make_params
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b, e = heads.rank_slice(n_heads, world, rank)
        params = make_params(head_base=b)
        # what every rank runs, gathered on every rank
        mine = torch.tensor([b, e, params.head_base], dtype=torch.int64)
        allv = [torch.zeros(3, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(allv, mine)
        q.put((rank, [tuple(int(x) for x in t) for t in allv]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("n_heads", [8, 40, 5])
def test_two_gloo_ranks_split_a_layer_by_heads(n_heads):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_heads_rank_main, args=(r, world, port, n_heads, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert res[0][1] == res[1][1]                   # both ranks see the same plan
    plan = res[0][1]
    covered = [h for (b, e, hb) in plan for h in range(b, e)]
    assert covered == list(range(n_heads))          # every head exactly once, in order
    for (b, e, hb) in plan:
        assert hb == b                              # random streams keyed by the global head index
    sizes = [e - b for (b, e, _) in plan]
    assert max(sizes) - min(sizes) <= 1


def test_head_slices_edge_cases():
    import sys
    sys.path.insert(0, ROOT)
    from free_clustered_block_b200 import heads
    assert heads.head_slices(3, 8) == [(0, 1), (1, 2), (2, 3)] + [(3, 3)] * 5
    assert heads.head_slices(0, 2) == [(0, 0), (0, 0)]
    assert heads.head_slices(40, 8) == [(5 * r, 5 * r + 5) for r in range(8)]
    with pytest.raises(ValueError):
        heads.rank_slice(4, 2, 2)
