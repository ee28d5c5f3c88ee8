"""The whole-backward call (sigattn_bwd) against the two separate backward
calls and against the fp64 oracle.

dQ and dK/dV depend only on Q, K, V and dO ("Better Models, Faster Training",
sec. 2B/2C: the sigmoid's Jacobian is diagonal, no row statistics of the
forward pass are needed), so the call runs the same two kernels with the
dK/dV kernel taking SMs as the dQ kernel's CTAs finish. Each output block
still has one owner and a fixed summation order, so the results must be
bit-identical to sigattn_bwd_dq + sigattn_bwd_dkdv; the oracle check pins
them independently, and the stream check makes sure later work in the same
stream sees all three outputs complete.
"""
import numpy as np
import pytest
import torch

import oracle
import sigmoid_attention_b200 as sa
from sigmoid_attention_b200 import workloads
from test_parity_gpu import BWD_REL, check_padded_zero, rel_l2

pytestmark = pytest.mark.gpu

CASES = [
    # (B, H, L, d, lengths, seed)
    (2, 2, 64, 64, [37, 64], 2001),
    (4, 2, 700, 64, [700, 129, 1, 0], 2002),             # ragged tail, n = 1, n = 0
    (3, 2, 520, 128, [520, 256, 255], 2003),
    (8, 1, 300, 128, [1, 127, 128, 129, 255, 256, 257, 300], 2004),
]


def _separate_and_fused(q, k, v, dout, lengths):
    dev = torch.device("cuda")
    B, H, L, d = q.shape
    qd, kd, vd, dod = (t.to(dev).contiguous() for t in (q, k, v, dout))
    lens = torch.as_tensor(lengths, dtype=torch.int32).to(dev)
    ws = sa.make_workspace(B, H, L, d, dev)
    sep = [torch.full_like(qd, float("nan")) for _ in range(3)]
    sa.sigattn_bwd_dq(qd, kd, vd, dod, sep[0], lens, ws)
    sa.sigattn_bwd_dkdv(qd, kd, vd, dod, sep[1], sep[2], lens, ws)
    fused = [torch.full_like(qd, float("nan")) for _ in range(3)]
    sa.sigattn_bwd(qd, kd, vd, dod, *fused, lens, ws)
    assert sa.sigattn_read_error(ws) == (0, 0)
    return sep, fused


@pytest.mark.parametrize("B,H,L,d,lengths,seed", CASES)
def test_fused_equals_separate_calls_and_oracle(B, H, L, d, lengths, seed):
    q, k, v, dout = workloads.make_inputs(B, H, L, d, seed)
    sep, fused = _separate_and_fused(q, k, v, dout, lengths)
    for name, a, b in zip(("dq", "dk", "dv"), sep, fused):
        assert torch.equal(a, b), name  # bit-identical (NaN poison would also fail here)
    refs = oracle.backward(q, k, v, dout, lengths)
    for name, got, ref in zip(("dq", "dk", "dv"), fused, refs):
        got = got.float().cpu()
        assert torch.isfinite(got).all(), name
        check_padded_zero(got, lengths)
        assert rel_l2(got, ref) <= BWD_REL, (name, rel_l2(got, ref))


@pytest.mark.parametrize("name", ["long_8k", "scrna_ragged"])
def test_fused_equals_separate_calls_on_workloads(name):
    # few work items per SM: the dK/dV kernel really starts beside the dQ kernel
    w = workloads.WORKLOADS[name]
    q, k, v, dout, lens = workloads.workload_inputs(w)
    sep, fused = _separate_and_fused(q, k, v, dout, lens.numpy())
    for label, a, b in zip(("dq", "dk", "dv"), sep, fused):
        assert torch.equal(a, b), label


def test_fused_repeatable_and_complete_for_the_stream():
    # Outputs poisoned with NaN, the call on a side stream, and a reduction of
    # all three outputs enqueued right after it on the same stream: the sums
    # must be those of the synchronised results.
    w = workloads.WORKLOADS["long_8k"]
    q, k, v, dout, lens = workloads.workload_inputs(w)
    dev = torch.device("cuda")
    qd, kd, vd, dod, ld = (t.to(dev) for t in (q, k, v, dout, lens))
    ws = sa.make_workspace(w.B, w.H, w.L, w.d, dev)
    side = torch.cuda.Stream()
    sums = []
    outs = []
    for _ in range(3):
        out = [torch.full_like(qd, float("nan")) for _ in range(3)]
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            sa.sigattn_bwd(qd, kd, vd, dod, *out, ld, ws, stream=side)
            sums.append(torch.stack([t.float().sum() for t in out]))
        torch.cuda.current_stream().wait_stream(side)
        outs.append(out)
    torch.cuda.synchronize()
    assert sa.sigattn_read_error(ws) == (0, 0)
    for s, out in zip(sums, outs):
        assert torch.isfinite(s).all()
        assert torch.equal(s, torch.stack([t.float().sum() for t in out]))
        for a, b in zip(out, outs[0]):
            assert torch.equal(a, b)


def test_fused_reports_bad_length_in_the_first_header():
    B, H, L, d = 2, 1, 256, 64
    q, k, v, dout = workloads.make_inputs(B, H, L, d, 2005)
    dev = torch.device("cuda")
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, dout))
    lens = torch.tensor([256, L + 5], dtype=torch.int32, device=dev)  # the second is out of range
    ws = sa.make_workspace(B, H, L, d, dev)
    out = [torch.full_like(qd, float("nan")) for _ in range(3)]
    sa.sigattn_bwd(qd, kd, vd, dod, *out, lens, ws)
    st, site = sa.sigattn_read_error(ws)
    assert st == 1 and site == -2, (st, site)
    for t in out:  # the bad sequence is treated as empty: all its rows are zero
        assert torch.equal(t[1], torch.zeros_like(t[1]))
        assert torch.isfinite(t[0].float()).all()


@pytest.mark.parametrize("name", ["long_8k", "scrna_ragged"])
def test_fused_varlen_equals_separate_varlen_and_padded(name):
    # the packed layout: the whole-backward call equals the two packed calls and
    # the padded whole-backward call on the same sequences, bit for bit
    w = workloads.WORKLOADS[name]
    q, k, v, dout, lens = workloads.workload_inputs(w)
    dev = torch.device("cuda")
    n = lens.tolist()
    pack = lambda t: torch.cat([t[b, :, :nb].permute(1, 0, 2) for b, nb in enumerate(n)]).contiguous().to(dev)
    qp, kp, vp, dp = (pack(t) for t in (q, k, v, dout))
    cu = torch.tensor([0] + list(np.cumsum(n)), dtype=torch.int32, device=dev)
    ws = sa.make_workspace(w.B, w.H, max(n), w.d, dev)
    sep = [torch.full_like(qp, float("nan")) for _ in range(3)]
    sa.sigattn_bwd_dq_varlen(qp, kp, vp, dp, sep[0], cu, max(n), ws)
    sa.sigattn_bwd_dkdv_varlen(qp, kp, vp, dp, sep[1], sep[2], cu, max(n), ws)
    fused = [torch.full_like(qp, float("nan")) for _ in range(3)]
    sa.sigattn_bwd_varlen(qp, kp, vp, dp, *fused, cu, max(n), ws)
    assert sa.sigattn_read_error(ws) == (0, 0)
    for label, a, b in zip(("dq", "dk", "dv"), sep, fused):
        assert torch.equal(a, b), label
    _, padded = _separate_and_fused(q, k, v, dout, lens.numpy())
    for label, a, b in zip(("dq", "dk", "dv"), padded, fused):
        assert torch.equal(pack(a.cpu()), b), label

