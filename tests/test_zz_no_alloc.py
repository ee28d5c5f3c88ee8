"""sigattn_fwd_noalloc: the forward entry point for callers that cannot
allocate device memory (it uses the library's fixed scratch array instead of a
caller workspace). Called through the C ABI with ctypes and compared with
sigattn_fwd on the same inputs, on two calls in a row with different shapes,
so the second call runs on whatever the first left in the shared array. Both
entry points run the same deterministic kernels on the same inputs, so their
outputs must be the same bits.

Collected last on purpose, so a run that stops at the first failure has
already run every other test."""
import ctypes

import pytest
import torch

import sigmoid_attention_b200 as sa
from sigmoid_attention_b200 import workloads

pytestmark = pytest.mark.gpu


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
        assert torch.equal(o, ref)  # same kernels, same inputs: the same bits


def test_noalloc_status_reports_this_call_only():
    """A call with an out-of-range length reports SIGATTN_ERR_INVALID_ARG in
    status_out and zeroes that sequence; the next, valid call starts from a
    cleared status and reports 0."""
    lib = sa.library()
    dev = torch.device("cuda")
    B, H, L, d = 2, 2, 256, 64
    q, k, v, _ = (t.to(dev) for t in workloads.make_inputs(B, H, L, d, 43))
    status = torch.full((1,), -7, dtype=torch.int32, device=dev)
    o = torch.full_like(q, float("nan"))
    bad = torch.tensor([L + 1, 200], dtype=torch.int32, device=dev)  # sequence 0 longer than Lmax
    assert _call_noalloc(lib, q, k, v, o, bad, status) == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 1
    assert torch.equal(o[0], torch.zeros_like(o[0]))
    good = torch.tensor([L, 200], dtype=torch.int32, device=dev)
    ref = torch.empty_like(q)
    sa.sigattn_fwd(q, k, v, ref, good, sa.make_workspace(B, H, L, d, dev))
    status.fill_(-7)
    assert _call_noalloc(lib, q, k, v, o, good, status) == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.equal(o, ref)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    lib = sa.library()
    fake = ctypes.c_void_p(1 << 20)  # aligned, never dereferenced: the size check comes first
    # 4096 * 64 * 1 work items of 16 bytes need 4 MiB of scratch, above the 1 MiB array
    st = lib.sigattn_fwd_noalloc(fake, fake, fake, fake, fake, 4096, 64, 128, 64, None, None)
    assert st == 2
    assert "scratch" in sa.sigattn_last_error()
    # a misaligned status pointer is rejected before anything is enqueued
    st = lib.sigattn_fwd_noalloc(fake, fake, fake, fake, fake, 1, 1, 128, 64, ctypes.c_void_p((1 << 20) + 2), None)
    assert st == 1
