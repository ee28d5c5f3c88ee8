"""Multi-rank plumbing of bench.py on CPU: two gloo ranks, max-over-ranks
timing and whole-job aggregation (units of all ranks over the slowest time)."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_seconds = 1.0 + rank  # rank 1 is the slow one
        t = bench.reduce_max(my_seconds, world, torch.device("cpu"))
        val = bench.whole_job_tflops(4e12, world, t)
        out[rank] = (t, val, bench._dist_env())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_max_time():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    for rank in range(world):
        t, val, env = res[rank]
        assert t == pytest.approx(2.0)                 # max over ranks
        assert val == pytest.approx(4e12 * 2 / 2.0 / 1e12)  # all ranks' units / slowest time
        assert env == (world, rank, rank)


def test_single_rank_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.whole_job_tflops(2e12, 1, 2.0) == pytest.approx(1.0)
