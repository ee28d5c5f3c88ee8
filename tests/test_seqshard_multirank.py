"""The host side of sequence-sharded attention on CPU: two gloo ranks, each
holding one key range, merge their partial outputs with seqshard.merge_partials_
(an all-reduce). Each rank's partial comes from the fp64 oracle restricted to
its keys (V zeroed outside the range for O; K zeroed outside it for dQ), so
the merged result must be the oracle's whole-sequence O and dQ."""
import os
import socket
import sys

import numpy as np
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
    import oracle
    from sigmoid_attention_b200 import seqshard, workloads

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, L, d = 2, 2, 300, 16
        lengths = [300, 190]
        q, k, v, dout = workloads.make_inputs(B, H, L, d, 71)
        begin, count = seqshard.key_range(rank, world, L)
        keep = torch.zeros(L, dtype=torch.bool)
        keep[begin:begin + count] = True
        v_in = torch.where(keep.view(1, 1, L, 1), v.float(), torch.zeros(()))
        k_in = torch.where(keep.view(1, 1, L, 1), k.float(), torch.zeros(()))
        o_part = torch.from_numpy(oracle.forward(q, k, v_in, lengths))
        dq_part = torch.from_numpy(oracle.backward(q, k_in, v, dout, lengths)[0])
        seqshard.merge_partials_(o_part)
        seqshard.merge_partials_(dq_part)
        o_ref = oracle.forward(q, k, v, lengths)
        dq_ref = oracle.backward(q, k, v, dout, lengths)[0]
        out[rank] = (float(np.abs(o_part.numpy() - o_ref).max()), float(np.abs(dq_part.numpy() - dq_ref).max()),
                     (begin, count))
    finally:
        dist.destroy_process_group()


def test_two_ranks_merge_partials_to_the_whole():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(180)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0][2] == (0, 256) and res[1][2] == (256, 44)
    for rank in range(world):
        o_err, dq_err, _ = res[rank]
        assert o_err <= 1e-12 and dq_err <= 1e-12


def test_key_ranges_tile_the_sequence():
    sys.path.insert(0, ROOT)
    from sigmoid_attention_b200 import seqshard

    for L in (1, 127, 128, 129, 300, 4096, 8191):
        for world in (1, 2, 3, 4, 8):
            ranges = [seqshard.key_range(r, world, L) for r in range(world)]
            pos = 0
            for begin, count in ranges:
                assert count >= 0 and begin == min(pos, L)
                if count > 0:
                    assert begin % 128 == 0
                pos = begin + count
            assert pos == L
    with pytest.raises(ValueError):
        seqshard.key_range(2, 2, 100)
