"""The N > 1 path of bench.py on the CPU: two gloo ranks, one process each.

Every rank runs its own problem (weak scaling, replicas only, no collective on
the data path); the only collectives are the barrier and the max-over-ranks
timing reduction, checked here with deliberately unequal per-rank timings.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w, r, local = bench._dist()
        assert (w, r, local) == (world, rank, rank)
        # rank r pretends its step took 10 + 5 r ms and its e2e 30 - r ms
        got = bench.max_over_ranks([10.0 + 5 * rank, 2.0 * rank, 30.0 - rank], world)
        dist.barrier()
        out.put((rank, got, bench.weak_scaling_value(world, 1e12, got[0])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_over_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, value in res:
        assert got == [15.0, 2.0, 30.0]          # slowest rank defines each time
        assert value == pytest.approx(2 * 1e12 / 15e-3 / 1e12)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5], 1) == [1.5, 2.5]
    assert bench.weak_scaling_value(1, 4e12, 2.0) == pytest.approx(2000.0)
