"""Pins of the oracle's softmax counterpart (oracle.softmax_forward), the
reference for the softmax kernel that shares the sigmoid path's scheduler
("Better Models, Faster Training", sec. 4A compares the two at 25% padding).

Softmax attention over the valid keys j < n: O_i = sum_j e^{S_ij} V_j /
sum_j e^{S_ij} with S_ij = <Q_i, K_j>/sqrt(d); lse_i = ln sum_j e^{S_ij}.
Each pin would fail under a plausible mistake: the zero-query mean over the
valid keys (wrong key range, a padding leak), V = 1 giving rows that sum to 1
(a missing normalisation), the single-token case (an index slip), an
independent fp64 torch composition (a wrong scale, a transposed operand),
and padded inputs changing nothing, bit for bit.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from sigmoid_attention_b200 import workloads


@pytest.mark.parametrize("d", [16, 64])
def test_zero_query_gives_the_mean_of_valid_values(d):
    B, H, L = 2, 2, 40
    lengths = [37, 1]
    _, k, v, _ = workloads.make_inputs(B, H, L, d, 601)
    q = torch.zeros_like(k)
    o, lse = oracle.softmax_forward(q, k, v, lengths)
    for b, n in enumerate(lengths):
        mean = v[b, :, :n].double().mean(dim=1).numpy()  # every weight is 1/n
        np.testing.assert_allclose(o[b, :, :n], np.broadcast_to(mean[:, None, :], o[b, :, :n].shape), rtol=1e-13,
                                   atol=1e-15)
        np.testing.assert_allclose(lse[b, :, :n], math.log(n), rtol=0, atol=1e-13)
        assert not o[b, :, n:].any() and not lse[b, :, n:].any()


def test_ones_value_rows_sum_to_one():
    B, H, L, d = 1, 3, 50, 32
    q, k, _, _ = workloads.make_inputs(B, H, L, d, 602)
    o, _ = oracle.softmax_forward(q * 3, k, torch.ones_like(q), [45])
    np.testing.assert_allclose(o[0, :, :45], 1.0, rtol=0, atol=1e-13)
    assert not o[0, :, 45:].any()


def test_single_token_returns_its_value():
    B, H, L, d = 1, 2, 8, 16
    q, k, v, _ = workloads.make_inputs(B, H, L, d, 603)
    o, lse = oracle.softmax_forward(q, k, v, [1])
    np.testing.assert_array_equal(o[0, :, 0], v[0, :, 0].double().numpy())
    s00 = (q[0, :, 0].double() * k[0, :, 0].double()).sum(-1).numpy() / math.sqrt(d)
    np.testing.assert_allclose(lse[0, :, 0], s00, rtol=0, atol=1e-14)


@pytest.mark.parametrize("d", [8, 64])
def test_matches_an_independent_torch_composition(d):
    B, H, L = 3, 2, 33
    lengths = [33, 20, 5]
    q, k, v, _ = workloads.make_inputs(B, H, L, d, 604)
    o, lse = oracle.softmax_forward(q, k, v, lengths)
    qd, kd, vd = (t.double() for t in (q, k, v))
    s = torch.einsum("bhid,bhjd->bhij", qd, kd) / math.sqrt(d)
    n = torch.tensor(lengths).view(B, 1, 1, 1)
    idx = torch.arange(L)
    keymask = idx.view(1, 1, 1, L) < n
    rowmask = idx.view(1, 1, L, 1) < n
    p = torch.softmax(s.masked_fill(~keymask, float("-inf")), dim=-1)
    ref = torch.where(rowmask, p @ vd, torch.zeros(()))
    ref_lse = torch.where(rowmask[..., 0], torch.logsumexp(s.masked_fill(~keymask, float("-inf")), dim=-1),
                          torch.zeros(()))
    np.testing.assert_allclose(o, ref.numpy(), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=1e-12, atol=1e-13)


def test_padded_inputs_change_nothing():
    B, H, L, d = 2, 2, 30, 16
    lengths = [30, 11]
    q, k, v, _ = workloads.make_inputs(B, H, L, d, 605)
    base = oracle.softmax_forward(q, k, v, lengths)
    q2, k2, v2 = (t.clone() for t in (q, k, v))
    for t in (q2, k2, v2):
        t[1, :, 11:] = 1000.0
    other = oracle.softmax_forward(q2, k2, v2, lengths)
    for a, b in zip(base, other):
        np.testing.assert_array_equal(a, b)
