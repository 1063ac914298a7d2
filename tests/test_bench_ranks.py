"""bench.py's multi-rank logic on CPU: two gloo ranks, each with its own
timings; the reported time is the max over ranks and the value counts every
rank's tokens (weak scaling)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [10.0 + 5.0 * rank, 3.0 - rank]          # rank 1 slower in the first, faster in the second
        got = bench.reduce_over_ranks(local, world)
        value = bench.aggregate_value(world, 100, 32768 * 4, got[0])
        out[rank] = (got, value)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_max_and_sum_work():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        for r in range(2):
            got, value = out[r]
            assert got == [15.0, 3.0]
            assert value == pytest.approx(2 * 100 * 32768 * 4 / 0.015)


def test_single_rank_passes_through():
    import bench
    assert bench.reduce_over_ranks([1.5, 2.5], 1) == [1.5, 2.5]
    assert bench.aggregate_value(1, 10, 1000, 1.0) == pytest.approx(10 * 1000 / 1e-3)
