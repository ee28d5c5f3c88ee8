"""sigattn_fwd_noalloc: the forward entry point for callers that cannot
allocate device memory (it uses the library's fixed scratch array instead of a
caller workspace). Called through the C ABI with ctypes and compared with
sigattn_fwd on the same inputs, on two calls in a row with different shapes,
so the second call runs on whatever the first left in the shared array.

Collected last on purpose, so a run that stops at the first failure has
already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import sigmoid_attention_b200 as sa
from sigmoid_attention_b200 import workloads

pytestmark = pytest.mark.gpu

FWD_REL, FWD_ABS = 5e-3, 2e-2  # the forward tolerance of the parity tests


def _rel_l2(a, b):
    a, b = a.double(), b.double()
    return (torch.linalg.vector_norm(a - b) / torch.linalg.vector_norm(b).clamp_min(1e-300)).item()


def _call_noalloc(lib, q, k, v, o, lens, status):
    B, H, L, d = q.shape
    return lib.sigattn_fwd_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
        ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lens.data_ptr()), B, H, L, d,
        ctypes.c_void_p(status.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_workspace_entry_point_twice():
    lib = sa.library()
    dev = torch.device("cuda")
    cases = [(3, 2, 700, 64, [700, 129, 1], 41), (2, 4, 520, 128, [520, 300], 42)]
    for B, H, L, d, lengths, seed in cases:
        q, k, v, _ = (t.to(dev) for t in workloads.make_inputs(B, H, L, d, seed))
        lens = torch.tensor(lengths, dtype=torch.int32, device=dev)
        ref = torch.empty_like(q)
        sa.sigattn_fwd(q, k, v, ref, lens, sa.make_workspace(B, H, L, d, dev))
        o = torch.full_like(q, float("nan"))
        status = torch.full((1,), -7, dtype=torch.int32, device=dev)
        assert _call_noalloc(lib, q, k, v, o, lens, status) == 0, sa.sigattn_last_error()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.isfinite(o).all()
        assert _rel_l2(o.float(), ref.float()) <= FWD_REL
        assert (o.float() - ref.float()).abs().max().item() <= FWD_ABS
        for b, n in enumerate(lengths):  # padded rows are zero, as with the workspace path
            assert torch.equal(o[b, :, n:], torch.zeros_like(o[b, :, n:]))


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = sa.library()
    null = ctypes.c_void_p(0)
    # 4096 * 64 * 1 work items need 2 MiB of scratch, above the 1 MiB array
    st = lib.sigattn_fwd_noalloc(null, null, null, null, null, 4096, 64, 128, 64, null, null)
    assert st == 2
    assert "scratch" in sa.sigattn_last_error()
