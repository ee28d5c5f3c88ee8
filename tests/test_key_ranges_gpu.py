"""Key-range calls (the pieces of sequence-sharded attention) against the
fp64 oracle and against the whole-sequence calls.

Each weight stands on its own ("Better Models, Faster Training", sec. 2A: no
normalisation over the keys), so the forward and dQ over a set of key ranges
that tile [0, Lmax) must add up to the whole-sequence results, and the dK/dV
rows of a range are those of the whole call. The oracle gives each range's
own share too: O restricted to keys in R is the oracle's O with V zeroed
outside R, and dQ restricted to R is the oracle's dQ with K zeroed outside R
(those keys' terms dS_ij K_j vanish, the others are unchanged).
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import sigmoid_attention_b200 as sa
from sigmoid_attention_b200 import seqshard, workloads
from test_parity_gpu import BWD_REL, FWD_ABS, FWD_REL, rel_l2, run_gpu

pytestmark = pytest.mark.gpu

CASES = [
    # (B, H, L, d, lengths, seed, range boundaries)
    (3, 2, 700, 64, [700, 300, 129], 401, [0, 256, 700]),
    (3, 2, 700, 128, [700, 300, 129], 402, [0, 128, 512, 700]),
    (2, 2, 520, 128, [520, 77], 403, [0, 100, 333, 520]),        # boundaries not on 128-row blocks
    (4, 1, 300, 64, [1, 128, 129, 300], 404, [0, 150, 300]),
]


def _ranges(bounds):
    return list(zip(bounds[:-1], [b - a for a, b in zip(bounds[:-1], bounds[1:])]))


@pytest.mark.parametrize("B,H,L,d,lengths,seed,bounds", CASES)
def test_ranges_sum_to_the_whole_call(B, H, L, d, lengths, seed, bounds):
    q, k, v, dout = workloads.make_inputs(B, H, L, d, seed)
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, dout))
    lens = torch.tensor(lengths, dtype=torch.int32, device=dev)
    ws = sa.make_workspace(B, H, L, d, dev)
    o_sum = torch.zeros((B, H, L, d), dtype=torch.float64)
    dq_sum = torch.zeros((B, H, L, d), dtype=torch.float64)
    dk_parts, dv_parts = [], []
    for begin, count in _ranges(bounds):
        kr, vr = kd[:, :, begin:begin + count].contiguous(), vd[:, :, begin:begin + count].contiguous()
        o32 = torch.full((B, H, L, d), float("nan"), device=dev)
        dq32 = torch.full((B, H, L, d), float("nan"), device=dev)
        dkr, dvr = (torch.full_like(kr, float("nan")) for _ in range(2))
        sa.sigattn_fwd_partial(qd, kr, vr, o32, lens, begin, ws)
        sa.sigattn_bwd_dq_partial(qd, kr, vr, dod, dq32, lens, begin, ws)
        sa.sigattn_bwd_dkdv_range(qd, kr, vr, dod, dkr, dvr, lens, begin, ws)
        assert sa.sigattn_read_error(ws) == (0, 0)
        o32, dq32 = o32.double().cpu(), dq32.double().cpu()
        for t in (o32, dq32, dkr, dvr):
            assert torch.isfinite(t).all()
        # this range's share against the oracle
        keep = torch.zeros(L, dtype=torch.bool)
        keep[begin:begin + count] = True
        v_in = torch.where(keep.view(1, 1, L, 1), v.float(), torch.zeros(())).to(v.dtype)
        k_in = torch.where(keep.view(1, 1, L, 1), k.float(), torch.zeros(())).to(k.dtype)
        o_ref = oracle.forward(q, k, v_in, lengths)
        dq_ref = oracle.backward(q, k_in, v, dout, lengths)[0]
        if np.linalg.norm(o_ref) > 0:
            assert rel_l2(o32.numpy(), o_ref) <= FWD_REL, ("o range", begin, rel_l2(o32.numpy(), o_ref))
        if np.linalg.norm(dq_ref) > 0:
            assert rel_l2(dq32.numpy(), dq_ref) <= BWD_REL, ("dq range", begin, rel_l2(dq32.numpy(), dq_ref))
        for b, n in enumerate(lengths):  # rows past n, and every row of a sequence with no key here, are 0
            rows = n if min(max(n - begin, 0), count) > 0 else 0
            assert torch.equal(o32[b, :, rows:], torch.zeros_like(o32[b, :, rows:]))
            assert torch.equal(dq32[b, :, rows:], torch.zeros_like(dq32[b, :, rows:]))
            keys = min(max(n - begin, 0), count)
            assert torch.equal(dkr[b, :, keys:].float().cpu(), torch.zeros_like(dkr[b, :, keys:].float().cpu()))
        o_sum += o32
        dq_sum += dq32
        dk_parts.append(dkr)
        dv_parts.append(dvr)
    o_ref = oracle.forward(q, k, v, lengths)
    dq_ref, dk_ref, dv_ref = oracle.backward(q, k, v, dout, lengths)
    assert rel_l2(o_sum.numpy(), o_ref) <= FWD_REL
    assert np.abs(o_sum.numpy() - o_ref).max() <= FWD_ABS
    assert rel_l2(dq_sum.numpy(), dq_ref) <= BWD_REL
    dk = torch.cat(dk_parts, dim=2).float().cpu()
    dv = torch.cat(dv_parts, dim=2).float().cpu()
    assert rel_l2(dk.numpy(), dk_ref) <= BWD_REL and rel_l2(dv.numpy(), dv_ref) <= BWD_REL
    whole = run_gpu(q, k, v, dout, lengths)
    if all(b % 128 == 0 for b in bounds[:-1]):
        # the same 128-row blocks in the same order: the same bits as the whole call
        assert torch.equal(dk, whole[2]) and torch.equal(dv, whole[3])
    # the summed fp32 forward, rounded once, matches the whole call within bf16 rounding
    o_bf16 = torch.empty((B, H, L, d), dtype=torch.bfloat16, device=dev)
    sa.sigattn_cast_bf16(o_sum.float().to(dev), o_bf16)
    assert torch.equal(o_bf16.cpu(), o_sum.float().to(torch.bfloat16))  # round to nearest even, as torch
    assert rel_l2(o_bf16.float().cpu().numpy(), whole[0].numpy()) <= FWD_REL


def test_seqshard_functions_on_one_gpu():
    """seqshard.forward / backward with one rank holding every key equal the
    whole-sequence calls (no process group: the sum is over one rank)."""
    B, H, L, d = 2, 2, 384, 64
    lengths = [384, 200]
    q, k, v, dout = (t.cuda() for t in workloads.make_inputs(B, H, L, d, 405))
    lens = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    begin, count = seqshard.key_range(0, 1, L)
    assert (begin, count) == (0, L)
    o = seqshard.forward(q, k, v, lens, begin)
    dq, dk, dv = seqshard.backward(q, k, v, dout, lens, begin)
    ref = run_gpu(*(t.cpu() for t in (q, k, v, dout)), lengths)
    assert rel_l2(o.float().cpu().numpy(), ref[0].numpy()) <= 1e-3
    assert rel_l2(dq.float().cpu().numpy(), ref[1].numpy()) <= 1e-3
    assert torch.equal(dk.float().cpu(), ref[2]) and torch.equal(dv.float().cpu(), ref[3])


def test_bad_key_ranges_rejected_before_any_work():
    lib = sa.library()
    fake = ctypes.c_void_p(1 << 20)
    B, H, L, d = 1, 1, 256, 64
    ws = sa.make_workspace(B, H, L, d)
    wsp, wsn = ctypes.c_void_p(ws.data_ptr()), ws.numel()
    lens = torch.tensor([256], dtype=torch.int32, device="cuda")
    lp = ctypes.c_void_p(lens.data_ptr())
    for begin, count in ((-1, 10), (0, 0), (200, 100), (256, 1)):
        assert lib.sigattn_fwd_partial(fake, fake, fake, fake, lp, B, H, L, d, begin, count, wsp, wsn, None) == 1
        assert lib.sigattn_bwd_dq_partial(fake, fake, fake, fake, fake, lp, B, H, L, d, begin, count, wsp, wsn,
                                          None) == 1
        assert lib.sigattn_bwd_dkdv_range(fake, fake, fake, fake, fake, fake, lp, B, H, L, d, begin, count, wsp, wsn,
                                          None) == 1
    assert lib.sigattn_cast_bf16(fake, fake, 7, None) == 1
