"""Pins for the fp64 oracle: closed forms, special cases, invariants, finite
differences and an independent fp64 torch composition. CPU only.

Each test is chosen so that a plausible mistake in the oracle fails it:
a dropped/mis-signed bias or a log in the wrong base (zero-query closed form),
1/d instead of 1/sqrt(d) (single-token case), padding not applied on one side
(closed form, zero rows, invariance), a transposed operand or a dropped
P(1-P) factor in the backward pass (finite differences, torch autograd).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from sigmoid_attention_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_sigmoid_closed_points():
    g = json.load(open(GOLDEN))
    for pt in g["sigmoid_points"]:
        x = {"0": 0.0, "-ln 3": -math.log(3.0), "ln 3": math.log(3.0)}[pt["x"]]
        assert oracle.sigmoid(x) == pytest.approx(float(Fraction(pt["value"])), rel=1e-15)
    # symmetry sigma(x) + sigma(-x) = 1 and the derivative bound sigma' <= 1/4 (sec. 2B)
    xs = np.linspace(-30, 30, 2001)
    s = np.array([oracle.sigmoid(x) for x in xs])
    s_neg = np.array([oracle.sigmoid(-x) for x in xs])
    assert np.allclose(s + s_neg, 1.0, atol=1e-15)
    h = 1e-5
    deriv = np.array([(oracle.sigmoid(x + h) - oracle.sigmoid(x - h)) / (2 * h) for x in xs])
    assert deriv.max() <= float(Fraction(g["sigmoid_derivative_max"])) + 1e-9
    assert np.allclose(deriv, s * (1 - s), atol=1e-9)


@pytest.mark.parametrize("d", [64, 128])
def test_zero_query_closed_form(d):
    g = json.load(open(GOLDEN))
    ns = [c["n"] for c in g["zero_query_weights"] if c["n"] <= 300]
    B, H, L = len(ns), 2, 300
    q = np.zeros((B, H, L, d))
    k = _rand((B, H, L, d), 1)
    v = _rand((B, H, L, d), 2)
    o = oracle.forward(q, k, v, ns)
    for b, n in enumerate(ns):
        w = float(Fraction(next(c["weight"] for c in g["zero_query_weights"] if c["n"] == n)))
        for h in range(H):
            expect = v[b, h, :n].sum(axis=0) * w
            assert np.allclose(o[b, h, :n], expect[None, :], rtol=1e-12, atol=1e-13)
            assert np.all(o[b, h, n:] == 0.0)
            assert oracle.weight(q[b, h], k[b, h], n, 0, n - 1) == pytest.approx(w, rel=1e-14)


def test_zero_query_ones_value_row_sums():
    # V = 1: O_i is the row sum of the weights, n/(1+n) for Q = 0.
    L, d = 80, 64
    ns = [1, 37, 64, 80]
    q = np.zeros((4, 1, L, d))
    k = _rand((4, 1, L, d), 3)
    v = np.ones((4, 1, L, d))
    o = oracle.forward(q, k, v, ns)
    for b, n in enumerate(ns):
        assert np.allclose(o[b, 0, :n], n / (1.0 + n), rtol=1e-13)
        assert np.all(o[b, 0, n:] == 0.0)


@pytest.mark.parametrize("d", [64, 128])
def test_single_token(d):
    # n = 1: bias ln 1 = 0, so O_0 = sigma(<q,k>/sqrt(d)) v, written out by hand.
    L = 3
    q, k, v = _rand((1, 1, L, d), 4), _rand((1, 1, L, d), 5), _rand((1, 1, L, d), 6)
    o = oracle.forward(q, k, v, [1])
    s = sum(q[0, 0, 0, c] * k[0, 0, 0, c] for c in range(d)) / math.sqrt(d)
    p = 1.0 / (1.0 + math.exp(-s))
    assert np.allclose(o[0, 0, 0], p * v[0, 0, 0], rtol=1e-13)
    assert np.all(o[0, 0, 1:] == 0.0)


def test_empty_sequence_gives_zeros():
    q, k, v, g = (_rand((2, 2, 16, 64), s) for s in range(7, 11))
    o = oracle.forward(q, k, v, [0, 16])
    dq, dk, dv = oracle.backward(q, k, v, g, [0, 16])
    for t in (o, dq, dk, dv):
        assert np.all(t[0] == 0.0)
        assert np.any(t[1] != 0.0)


def test_padding_invariance():
    """Padded keys, values, queries and upstream gradients are ignored exactly."""
    B, H, L, d = 3, 2, 40, 64
    lens = [13, 40, 1]
    q, k, v, g = (_rand((B, H, L, d), s) for s in range(11, 15))
    o = oracle.forward(q, k, v, lens)
    grads = oracle.backward(q, k, v, g, lens)
    q2, k2, v2, g2 = (t.copy() for t in (q, k, v, g))
    for b, n in enumerate(lens):
        for t, s in ((q2, 20), (k2, 21), (v2, 22), (g2, 23)):
            t[b, :, n:] = 1e6 * _rand(t[b, :, n:].shape, s + b)
    assert np.array_equal(oracle.forward(q2, k2, v2, lens), o)
    for a, b_ in zip(oracle.backward(q2, k2, v2, g2, lens), grads):
        assert np.array_equal(a, b_)


def test_weights_elementwise_and_bounded():
    """Each weight depends only on its own score (diagonal Jacobian, sec. 2B):
    changing key l changes column l of P and nothing else. Weights lie in
    (0, 1) inside the valid square and are exactly 0 outside it."""
    L, d, n = 12, 64, 10
    q, k = _rand((L, d), 30), _rand((L, d), 31)
    P = np.array([[oracle.weight(q, k, n, i, j) for j in range(L)] for i in range(L)])
    assert np.all(P[:n, :n] > 0) and np.all(P[:n, :n] < 1)
    assert np.all(P[n:, :] == 0) and np.all(P[:, n:] == 0)
    assert np.all(P * (1 - P) <= 0.25)
    k2 = k.copy()
    k2[4] += 0.5
    P2 = np.array([[oracle.weight(q, k2, n, i, j) for j in range(L)] for i in range(L)])
    changed = P2 != P
    assert changed[:n, 4].all()
    changed[:, 4] = False
    assert not changed.any()


@pytest.mark.parametrize("n,L", [(4, 5), (5, 5), (1, 3)])
def test_backward_matches_central_differences(n, L):
    """dQ, dK, dV from the analytic backward vs central differences of
    loss = sum(O * G) computed with the oracle forward (fp64, h = 1e-6)."""
    d = 8
    q, k, v, g = (_rand((1, 1, L, d), s) for s in range(40, 44))
    dq, dk, dv = oracle.backward(q, k, v, g, [n])
    h = 1e-6

    def loss(qq, kk, vv):
        return float(np.sum(oracle.forward(qq, kk, vv, [n]) * g))

    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            fd[idx] = (loss(args_p["q"], args_p["k"], args_p["v"]) -
                       loss(args_m["q"], args_m["k"], args_m["v"])) / (2 * h)
        err = np.abs(fd - grad).max() / max(np.abs(grad).max(), 1e-30)
        assert err < 1e-7, (name, err)
        # padded rows of the gradient are exactly zero
        assert np.all(grad[0, 0, n:] == 0.0)


def _torch_reference(q, k, v, g, lens):
    """An independent fp64 composition with torch ops and autograd."""
    q, k, v, g = (torch.tensor(t, dtype=torch.float64, requires_grad=True) for t in (q, k, v, g))
    B, H, L, d = q.shape
    idx = torch.arange(L)
    n = torch.tensor(lens, dtype=torch.float64)
    valid = idx[None, :] < torch.tensor(lens)[:, None]  # [B, L]
    mask = valid[:, None, :, None] & valid[:, None, None, :]  # [B,1,L,L]
    bias = -torch.log(torch.clamp(n, min=1.0))[:, None, None, None]
    s = torch.matmul(q, k.transpose(-1, -2)) / math.sqrt(d) + bias
    p = torch.where(mask, torch.sigmoid(s), torch.zeros_like(s))
    o = torch.matmul(p, v)
    o.backward(g.detach())
    return o.detach().numpy(), q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("d", [64, 128])
def test_matches_torch_fp64_autograd(d):
    B, H, L = 3, 2, 70
    lens = [70, 33, 1]
    q, k, v, g = (_rand((B, H, L, d), s) for s in range(50, 54))
    o_t, dq_t, dk_t, dv_t = _torch_reference(q, k, v, g, lens)
    o = oracle.forward(q, k, v, lens)
    dq, dk, dv = oracle.backward(q, k, v, g, lens)
    for a, b in ((o, o_t), (dq, dq_t), (dk, dk_t), (dv, dv_t)):
        assert np.allclose(a, b, rtol=1e-10, atol=1e-12)
        for bi, n in enumerate(lens):
            assert np.all(a[bi, :, n:] == 0.0)


def test_sampled_rows_equal_full_outputs():
    B, H, L, d = 2, 3, 50, 64
    lens = [50, 17]
    q, k, v, g = (_rand((B, H, L, d), s) for s in range(60, 64))
    o = oracle.forward(q, k, v, lens)
    dq, dk, dv = oracle.backward(q, k, v, g, lens)
    rng = np.random.default_rng(0)
    bh = rng.integers(0, B * H, 25)
    row = rng.integers(0, L, 25)
    for which, full in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv)):
        got = oracle.rows(which, q, k, v, g, lens, bh, row)
        expect = full.reshape(B * H, L, d)[bh, row]
        assert np.array_equal(got, expect), which


@pytest.mark.parametrize("block", [64, 128, 256])
def test_tile_enumeration_brute_force(block):
    H, L = 3, 1000
    lens = [0, 1, block - 1, block, block + 1, 999, 1000, 2 * block]
    got = oracle.tiles(lens, H, L, block)
    expect = []
    for b, n in enumerate(lens):
        for h in range(H):
            for m in range((L + block - 1) // block):
                rows_in_block = range(m * block, min((m + 1) * block, L))
                if any(r < n for r in rows_in_block):
                    expect.append((b, h, m))
    assert [tuple(t) for t in got.tolist()] == expect
    assert len(got) == sum(H * ((n + block - 1) // block) for n in lens)


def test_workload_lengths_recipes():
    w = workloads.WORKLOADS
    assert list(w["tiny"].lengths()) == [37, 64]
    assert (w["dense_d128"].lengths() == 4096).all()
    sc = w["scrna_ragged"].lengths()
    assert sc.min() >= 256 and sc.max() <= 2048 and len(sc) == 8
    lg = w["long_8k"].lengths()
    assert lg.min() >= 1024 and lg.max() <= 8192
    assert (w["pad_sweep_p00"].lengths() == 4096).all()
    p75 = w["pad_sweep_p75"].lengths()
    assert p75.min() >= 1 and p75.max() <= 2048
    # inputs are reproducible from the seed
    a = workloads.make_inputs(1, 1, 8, 64, 7)
    b = workloads.make_inputs(1, 1, 8, 64, 7)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
