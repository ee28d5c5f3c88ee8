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


def _bench_env():
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "LOCAL_RANK", "WORLD_SIZE", "MASTER_ADDR",
                                                            "MASTER_PORT")}
    env["CUDA_VISIBLE_DEVICES"] = ""
    return env


def test_gpus_flag_starts_that_many_ranks():
    """`bench.py --gpus 2` without a launcher starts two ranks itself; the
    line rank 0 prints counts both (the reference arm needs no GPU)."""
    import json
    import subprocess

    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
                          "--workload", "tiny", "--steps", "3", "--warmup", "3"], cwd=ROOT, env=_bench_env(),
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    assert json.loads(lines[0])["n_gpus"] == 2


def test_gpus_flag_must_match_the_launcher():
    import subprocess

    env = _bench_env()
    env.update(WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference",
                          "--workload", "tiny", "--steps", "3", "--warmup", "3"], cwd=ROOT, env=env,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode != 0
    assert "WORLD_SIZE=1" in out.stderr
