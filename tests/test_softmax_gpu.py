"""The softmax counterpart (sigattn_softmax_fwd) against the fp64 oracle's
softmax attention over the valid keys (oracle.softmax_forward).

It shares the sigmoid forward's plan, scheduler, loads and MMAs, so that the
two can be timed on equal terms ("Better Models, Faster Training", sec. 4A,
compares the sigmoid kernel with softmax attention at 25% padding). Tolerances
are the sigmoid forward's: rel-L2 <= 5e-3 and max-abs <= 2e-2 against fp64
(P and O are rounded to bf16 once each). Cases: ragged lengths across several
tiles, single-token and empty sequences, scores scaled by 4 (peaked rows: the
running maximum moves and O is rescaled), a slice of the 25%-padded sweep
workload, padded inputs that must change nothing, and repeat runs that must
give the same bits.
"""
import numpy as np
import pytest
import torch

import oracle
import sigmoid_attention_b200 as sa
from sigmoid_attention_b200 import workloads
from test_parity_gpu import FWD_ABS, FWD_REL, rel_l2

pytestmark = pytest.mark.gpu


def run_softmax(q, k, v, lengths):
    dev = torch.device("cuda")
    B, H, L, d = q.shape
    qd, kd, vd = (t.to(dev).contiguous() for t in (q, k, v))
    lens = torch.as_tensor(np.asarray(lengths), dtype=torch.int32).to(dev)
    ws = sa.make_workspace(B, H, L, d, dev)
    o = torch.full_like(qd, float("nan"))
    sa.sigattn_softmax_fwd(qd, kd, vd, o, lens, ws)
    assert sa.sigattn_read_error(ws) == (0, 0)
    return o.float().cpu()


def check(q, k, v, lengths):
    o = run_softmax(q, k, v, lengths)
    assert torch.isfinite(o).all()
    for b, n in enumerate(np.asarray(lengths)):
        assert torch.equal(o[b, :, int(n):], torch.zeros_like(o[b, :, int(n):]))
    ref, _ = oracle.softmax_forward(q, k, v, lengths)
    assert rel_l2(o, ref) <= FWD_REL, rel_l2(o, ref)
    assert np.abs(o.numpy() - ref).max() <= FWD_ABS
    return o


CASES = [
    (2, 2, 64, [37, 64], 701),
    (4, 2, 700, [700, 129, 1, 0], 702),
    (8, 1, 300, [1, 127, 128, 129, 255, 256, 257, 300], 703),
    (2, 3, 200, [200, 77], 704),
    (1, 2, 1024, [1024], 705),
]


@pytest.mark.parametrize("B,H,L,lengths,seed", CASES)
def test_softmax_small_cases(B, H, L, lengths, seed):
    q, k, v, _ = workloads.make_inputs(B, H, L, 64, seed)
    check(q, k, v, lengths)


@pytest.mark.parametrize("scale", [4.0, 8.0])
def test_softmax_peaked_rows_rescale(scale):
    # Q, K scaled (exact in bf16): scores spread over tens of units, so the
    # row maximum keeps rising across key blocks and O is rescaled.
    B, H, L = 2, 2, 900
    lengths = [900, 513]
    q, k, v, _ = workloads.make_inputs(B, H, L, 64, 706)
    check(q * scale, k, v, lengths)


def test_softmax_slice_of_the_padding_sweep():
    w = workloads.WORKLOADS["pad_sweep_p25"]
    q, k, v, _, lens = workloads.workload_inputs(w)
    sl = slice(0, 2)
    check(q[sl, :2].contiguous(), k[sl, :2].contiguous(), v[sl, :2].contiguous(), lens[sl].numpy())


def test_softmax_padded_inputs_ignored_and_deterministic():
    B, H, L = 3, 2, 300
    lengths = [300, 140, 17]
    q, k, v, _ = workloads.make_inputs(B, H, L, 64, 707)
    base = run_softmax(q, k, v, lengths)
    assert torch.equal(base, run_softmax(q, k, v, lengths))
    q2, k2, v2 = (t.clone() for t in (q, k, v))
    g = torch.Generator().manual_seed(9)
    for b, n in enumerate(lengths):
        for t in (q2, k2, v2):
            t[b, :, n:] = (100 * torch.randn(t[b, :, n:].shape, generator=g)).to(t.dtype)
    assert torch.equal(base, run_softmax(q2, k2, v2, lengths))


def test_softmax_head_size_128_unsupported():
    q = torch.zeros((1, 1, 128, 128), dtype=torch.bfloat16, device="cuda")
    lens = torch.tensor([128], dtype=torch.int32, device="cuda")
    ws = sa.make_workspace(1, 1, 128, 128)
    with pytest.raises(sa.SigattnError):
        sa.sigattn_softmax_fwd(q, q, q, torch.empty_like(q), lens, ws)
