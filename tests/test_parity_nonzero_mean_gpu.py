"""GPU parity with values whose mean is not zero.

With V drawn i.i.d. N(0,1) the per-weight errors of the sigmoid cancel in
O_i = sum_j P_ij V_j, so a sigmoid whose error has a consistent sign near
sigma ~ 1/n would go unseen. Here V = 1 (O_i is the row sum of the weights) and
V = |N(0,1)|, with Q, K i.i.d. N(0,1), and a zero-query case whose every
weight is exactly 1/(1+n) (the bias -ln n of "Better Models, Faster Training:
Sigmoid Attention for single-cell Foundation Models", sec. 2A), so that
O_i = sum_{j<n} V_j / (1+n) in closed form and the sigmoid's error at one
point enters every weight with the same sign.

Sizes n = 4096, 8192 and 65536 tokens (the weights then sit near 2.4e-4,
1.2e-4 and 1.5e-5) at d = 64 and 128. Tolerances are the parity tests' own,
against fp64: O rel-L2 <= 5e-3 and max-abs <= 2e-2, dQ/dK/dV rel-L2 <= 1e-2.
"""
import numpy as np
import pytest
import torch

import oracle
from sigmoid_attention_b200 import workloads
from test_parity_gpu import BWD_REL, FWD_ABS, FWD_REL, rel_l2, run_gpu

pytestmark = pytest.mark.gpu


def _inputs(n, d, values, query, seed):
    q, k, v, dout = workloads.make_inputs(1, 1, n, d, seed)
    if values == "ones":
        v = torch.ones_like(v)
    elif values == "abs":
        v = v.abs()
    if query == "zero":
        q = torch.zeros_like(q)
    return q, k, v, dout


CASES = [(n, d, values, query)
         for n in (4096, 8192, 65536) for d in (64, 128)
         for values, query in (("ones", "normal"), ("abs", "normal"), ("ones", "zero"))]


@pytest.mark.parametrize("n,d,values,query", CASES)
def test_nonzero_mean_values(n, d, values, query):
    seed = 500 + n % 997 + d
    q, k, v, dout = _inputs(n, d, values, query, seed)
    lens = np.array([n], dtype=np.int32)
    o, dq, dk, dv = run_gpu(q, k, v, dout, lens)
    for t in (o, dq, dk, dv):
        assert torch.isfinite(t).all()
    rng = np.random.default_rng(seed)
    row = np.concatenate([[0, n - 1], rng.integers(0, n, 14)])
    bh = np.zeros_like(row)
    if query == "zero":
        # every weight is 1/(1+n): O_i = sum_j V_j / (1+n) for every valid row i
        expect = v[0, 0].double().sum(dim=0).numpy() / (1.0 + n)
        got = o.reshape(n, d).numpy().astype(np.float64)
        err = rel_l2(got, np.broadcast_to(expect, got.shape))
        assert err <= FWD_REL, ("o closed form", err)
        assert np.abs(got - expect).max() <= FWD_ABS
    for name, got, tol in (("o", o, FWD_REL), ("dq", dq, BWD_REL), ("dk", dk, BWD_REL), ("dv", dv, BWD_REL)):
        ref = oracle.rows(name, q, k, v, dout, lens, bh, row)
        g = got.reshape(n, d)[row].numpy()
        err = rel_l2(g, ref)
        assert err <= tol, (name, err)
        if name == "o":
            assert np.abs(g - ref).max() <= FWD_ABS
