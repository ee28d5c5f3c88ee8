"""GPU checks of the packed ("varlen") entry points: sequences stored back to
back as [total, H, d] with cumulative offsets cu_seqlens.

The packed calls run the same tiles, in the same order, through the same
tensor-core products as the padded calls; the rows past a sequence's end that a
tile reads belong to the next sequence instead of padding, and enter only as
0 * value. So on the valid rows the packed results must equal the padded ones
bit for bit, and the padded path is itself checked against the fp64 oracle
(test_parity_gpu.py). One case is also compared with the oracle directly.
"""
import numpy as np
import pytest
import torch

import oracle
import sigmoid_attention_b200 as sa
from sigmoid_attention_b200 import workloads

pytestmark = pytest.mark.gpu

FWD_REL, FWD_ABS, BWD_REL = 5e-3, 2e-2, 1e-2


def rel_l2(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)


def pack(t, lengths, lead=0, tail=0):
    """[B, H, L, d] -> [lead + sum(n) + tail, H, d] and cu_seqlens. The lead and
    tail rows belong to no sequence; they hold large finite values (the last
    sequence's last tile reads them, and they must not matter)."""
    B, H, L, d = t.shape
    g = torch.Generator().manual_seed(9)
    parts = [(100 * torch.randn(lead, H, d, generator=g)).to(t.dtype)]
    cu = [lead]
    for b, n in enumerate(lengths):
        parts.append(t[b, :, :n].permute(1, 0, 2))
        cu.append(cu[-1] + int(n))
    parts.append((100 * torch.randn(tail, H, d, generator=g)).to(t.dtype))
    return torch.cat(parts).contiguous(), torch.tensor(cu, dtype=torch.int32)


def unpack(p, cu, B, L):
    """[total, H, d] -> [B, H, L, d] with zeros past each sequence's end."""
    _, H, d = p.shape
    out = torch.zeros(B, H, L, d, dtype=p.dtype)
    for b in range(B):
        s, e = int(cu[b]), int(cu[b + 1])
        out[b, :, : e - s] = p[s:e].permute(1, 0, 2)
    return out


def run_padded(q, k, v, dout, lengths):
    dev = torch.device("cuda")
    B, H, L, d = q.shape
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, dout))
    lens = torch.as_tensor(np.asarray(lengths), dtype=torch.int32).to(dev)
    ws = sa.make_workspace(B, H, L, d, dev)
    o, dq, dk, dv = (torch.empty_like(qd) for _ in range(4))
    sa.sigattn_fwd(qd, kd, vd, o, lens, ws)
    sa.sigattn_bwd_dq(qd, kd, vd, dod, dq, lens, ws)
    sa.sigattn_bwd_dkdv(qd, kd, vd, dod, dk, dv, lens, ws)
    assert sa.sigattn_read_error(ws) == (0, 0)
    return [t.cpu() for t in (o, dq, dk, dv)]


def run_packed(q, k, v, dout, lengths, lead=0, tail=0):
    """Packed calls on the same sequences; returns unpacked results plus the raw packed outputs."""
    dev = torch.device("cuda")
    B, H, L, d = q.shape
    packed = [pack(t, lengths, lead, tail) for t in (q, k, v, dout)]
    cu = packed[0][1]
    qp, kp, vp, dop = (p[0].to(dev) for p in packed)
    cud = cu.to(dev)
    maxlen = max(1, int(np.max(lengths)))
    ws = sa.make_workspace(B, H, maxlen, d, dev)
    o, dq, dk, dv = (torch.full_like(qp, float("nan")) for _ in range(4))
    sa.sigattn_fwd_varlen(qp, kp, vp, o, cud, maxlen, ws)
    sa.sigattn_bwd_dq_varlen(qp, kp, vp, dop, dq, cud, maxlen, ws)
    sa.sigattn_bwd_dkdv_varlen(qp, kp, vp, dop, dk, dv, cud, maxlen, ws)
    assert sa.sigattn_read_error(ws) == (0, 0)
    raw = [t.cpu() for t in (o, dq, dk, dv)]
    return [unpack(t, cu, B, L) for t in raw], raw, cu


CASES = [
    # (B, H, L, d, lengths, seed)
    (4, 2, 700, 64, [700, 129, 1, 0], 41),
    (3, 2, 520, 128, [520, 256, 255], 42),
    (8, 1, 300, 64, [1, 127, 128, 129, 255, 256, 257, 300], 43),
    (8, 1, 300, 128, [1, 127, 128, 129, 255, 256, 257, 300], 44),
    (2, 3, 1000, 64, [1000, 37], 45),
]


@pytest.mark.parametrize("B,H,L,d,lengths,seed", CASES)
def test_packed_equals_padded_bitwise(B, H, L, d, lengths, seed):
    q, k, v, dout = workloads.make_inputs(B, H, L, d, seed)
    padded = run_padded(q, k, v, dout, lengths)
    packed, raw, _ = run_packed(q, k, v, dout, lengths)
    for name, a, b in zip(("o", "dq", "dk", "dv"), padded, packed):
        assert torch.equal(a, b), name
    for t in raw:
        assert torch.isfinite(t.float()).all()  # every packed row belongs to a sequence and was written


def test_packed_matches_oracle():
    B, H, L, d = 3, 2, 400, 64
    lengths = [400, 211, 64]
    q, k, v, dout = workloads.make_inputs(B, H, L, d, 46)
    (o, dq, dk, dv), _, _ = run_packed(q, k, v, dout, lengths)
    o_ref = oracle.forward(q, k, v, lengths)
    dq_ref, dk_ref, dv_ref = oracle.backward(q, k, v, dout, lengths)
    assert rel_l2(o.float(), o_ref) <= FWD_REL
    assert np.abs(o.float().numpy() - o_ref).max() <= FWD_ABS
    for got, ref in ((dq, dq_ref), (dk, dk_ref), (dv, dv_ref)):
        assert rel_l2(got.float(), ref) <= BWD_REL


def test_rows_outside_every_sequence_are_untouched():
    B, H, L, d = 3, 2, 300, 128
    lengths = [300, 90, 129]
    q, k, v, dout = workloads.make_inputs(B, H, L, d, 47)
    padded = run_padded(q, k, v, dout, lengths)
    packed, raw, cu = run_packed(q, k, v, dout, lengths, lead=5, tail=7)
    for a, b in zip(padded, packed):
        assert torch.equal(a, b)
    for t in raw:
        assert torch.isnan(t[:5].float()).all() and torch.isnan(t[-7:].float()).all()
        assert torch.isfinite(t[5:-7].float()).all()


def test_invalid_bounds_flag_error_and_skip_the_sequence():
    dev = torch.device("cuda")
    H, d = 2, 64
    q, k, v = (torch.randn(100, H, d, dtype=torch.float32).to(torch.bfloat16).to(dev) for _ in range(3))
    cu = torch.tensor([0, 40, 120], dtype=torch.int32, device=dev)  # sequence 1 ends past total = 100
    ws = sa.make_workspace(2, H, 80, d, dev)
    o = torch.full_like(q, float("nan"))
    sa.sigattn_fwd_varlen(q, k, v, o, cu, 80, ws)
    st, site = sa.sigattn_read_error(ws)
    assert st == 1 and site == -2
    assert torch.isfinite(o[:40].float()).all() and torch.isnan(o[40:].float()).all()
    # sequence 0 alone, through the padded call, gives the same bits
    q0, k0, v0 = (t[:40].permute(1, 0, 2).unsqueeze(0).contiguous() for t in (q, k, v))
    ref = torch.empty_like(q0)
    sa.sigattn_fwd(q0, k0, v0, ref, torch.tensor([40], dtype=torch.int32, device=dev),
                   sa.make_workspace(1, H, 40, d, dev))
    assert torch.equal(o[:40].permute(1, 0, 2).unsqueeze(0), ref)


@pytest.mark.parametrize("name", ["scrna_ragged", "pad_sweep_p50", "long_8k"])
def test_full_size_workload_packed_equals_padded(name):
    w = workloads.WORKLOADS[name]
    q, k, v, dout, lens = workloads.workload_inputs(w)
    lengths = lens.numpy()
    padded = run_padded(q, k, v, dout, lengths)
    packed, _, _ = run_packed(q, k, v, dout, lengths)
    for nm, a, b in zip(("o", "dq", "dk", "dv"), padded, packed):
        assert torch.equal(a, b), (name, nm)


def test_varlen_autograd_matches_direct_calls():
    B, H, L, d = 3, 2, 300, 64
    lengths = [300, 90, 129]
    q, k, v, dout = workloads.make_inputs(B, H, L, d, 48)
    (_, raw, cu) = run_packed(q, k, v, dout, lengths)
    dev = torch.device("cuda")
    qp, kp, vp, dop = (pack(t, lengths)[0].to(dev) for t in (q, k, v, dout))
    qp, kp, vp = (t.requires_grad_(True) for t in (qp, kp, vp))
    o = sa.sigmoid_attention_varlen(qp, kp, vp, cu.to(dev), max(lengths))
    o.backward(dop)
    for got, ref in zip((o.detach(), qp.grad, kp.grad, vp.grad), raw):
        assert torch.equal(got.cpu(), ref)
