"""The sigmoid as the kernels evaluate it, pinned to the exact function.

"Better Models, Faster Training: Sigmoid Attention for single-cell Foundation
Models", sec. 2A: the weight of score s in a sequence of n tokens is
sigma(s / sqrt(d) - ln n); sec. 2B: its derivative is sigma (1 - sigma).
sigattn_eval_sigmoid runs the kernels' own code for both on any scores; here
it is compared, element by element, with the fp64 functions of the same fp32
scores. The bias puts typical weights near 1/n, far in the lower tail, so the
tail is where a relative error would shift every output of a row alike: it
gets a bound 50 times tighter than the rest of the line.

The second test is end to end: with Q = 0 every weight of a row is
sigma(-ln n) = 1/(1+n) exactly, so with V = 1 each valid row of O equals
n/(1+n). Twenty-four lengths between 1000 and 65536 run in one call, so the
bias takes many values across the range where weights are small.
"""
import math

import numpy as np
import pytest
import torch

import sigmoid_attention_b200 as sa
from sigmoid_attention_b200 import workloads

pytestmark = pytest.mark.gpu


def _sigma_and_slope(x):
    """fp64 sigma(x) and sigma'(x), written without cancellation in either tail."""
    a = np.exp(-np.abs(x))
    lower = a / (1.0 + a)            # sigma(-|x|)
    upper = 1.0 / (1.0 + a)          # sigma(|x|)
    sig = np.where(x < 0, lower, upper)
    return sig, lower * upper


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n", [1, 37, 4096, 8192, 50419, 1 << 20])
def test_sigmoid_matches_exact_function(d, n):
    scale = 1.0 / math.sqrt(d)
    # scores giving x = s/sqrt(d) - ln n over [-100, 60]
    x_target = np.linspace(-100.0, 60.0, 400001)
    s = ((x_target + math.log(n)) / scale).astype(np.float32)
    p, slope = sa.sigattn_eval_sigmoid(torch.from_numpy(s).cuda(), d, n)
    p, slope = p.cpu().numpy().astype(np.float64), slope.cpu().numpy().astype(np.float64)
    x = s.astype(np.float64) * scale - math.log(n)
    ref, ref_slope = _sigma_and_slope(x)
    assert np.isfinite(p).all() and np.isfinite(slope).all()
    # sigma' <= 1/4 (sec. 2B); the route makes sigma(0) = 1/2 exact, so only fp32 rounding may exceed it
    assert (p >= 0).all() and (p <= 1).all() and (slope >= 0).all() and (slope <= 0.25 + 1e-6).all()
    live = ref > 1e-30                 # below ~1e-38 the exp2 flushes to zero; such weights are 0
    rel = np.abs(p[live] / ref[live] - 1.0)
    assert rel.max() <= 1e-3, (float(rel.max()), float(x[live][np.argmax(rel)]))
    tail = live & (x < -5.0)
    rel_tail = np.abs(p[tail] / ref[tail] - 1.0)
    assert rel_tail.max() <= 2e-5, (float(rel_tail.max()), float(x[tail][np.argmax(rel_tail)]))
    assert np.abs(p[~live]).max(initial=0.0) <= 1e-30
    live_s = ref_slope > 1e-30
    rel_s = np.abs(slope[live_s] / ref_slope[live_s] - 1.0)
    assert rel_s.max() <= 2e-3, (float(rel_s.max()), float(x[live_s][np.argmax(rel_s)]))


def test_zero_query_closed_form_over_many_lengths():
    d, H = 64, 1
    lengths = np.unique(np.round(np.exp(np.linspace(math.log(1000), math.log(65536), 24)))).astype(np.int32)
    B, L = len(lengths), int(lengths.max())
    _, k, _, _ = workloads.make_inputs(B, H, L, d, 301)
    dev = torch.device("cuda")
    q = torch.zeros((B, H, L, d), dtype=torch.bfloat16, device=dev)
    v = torch.ones((B, H, L, d), dtype=torch.bfloat16, device=dev)
    o = torch.full_like(q, float("nan"))
    lens = torch.from_numpy(lengths).to(dev)
    ws = sa.make_workspace(B, H, L, d, dev)
    sa.sigattn_fwd(q, k.to(dev), v, o, lens, ws)
    assert sa.sigattn_read_error(ws) == (0, 0)
    for b, n in enumerate(lengths.tolist()):
        got = o[b, 0, :n].double().cpu().numpy()
        expect = n / (1.0 + n)
        err = np.abs(got / expect - 1.0)
        # P = 1/(1+n) and O are each rounded to bf16 once: <= 2^-9 apiece
        assert err.max() <= 5e-3, (n, float(err.max()))
        assert torch.equal(o[b, 0, n:], torch.zeros_like(o[b, 0, n:]))
