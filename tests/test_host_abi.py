"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function the header declares, rejects bad arguments before touching the
device, and its host statement of the tile schedule enumerates exactly the
oracle's active tiles, longest sequence first."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import oracle
import sigmoid_attention_b200 as sa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sigattn.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"SIGATTN_API\s+[\w\s\*]+?\b(sigattn_\w+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 10
    lib = ctypes.CDLL(sa.library_path())
    for name in names:
        assert hasattr(lib, name), name


def test_status_strings_and_sizes():
    assert sa.sigattn_version() == 100
    assert sa.sigattn_status_str(0) == "ok"
    assert "timed out" in sa.sigattn_status_str(4)
    assert [sa.sigattn_block_rows(k) for k in (0, 1, 2)] == [256, 128, 128]
    assert sa.sigattn_block_rows(3) == -1
    # header + one 16-byte entry per possible 128-row item
    assert sa.sigattn_workspace_size(4, 16, 4096, 128) == 256 + 16 * 4 * 16 * 32
    assert sa.sigattn_workspace_size(2, 2, 64, 64) == 256 + 16 * 4
    assert sa.sigattn_workspace_size(1, 1, 1, 96) == 0      # unsupported head size
    assert sa.sigattn_workspace_size(0, 1, 1, 64) == 0
    assert sa.sigattn_workspace_size(5000, 1, 1, 64) == 0   # beyond SIGATTN_MAX_BATCH
    # the whole-backward call holds two work lists, each rounded up to 256 bytes
    assert sa.sigattn_bwd_workspace_size(4, 16, 4096, 128) == 2 * (256 + 16 * 4 * 16 * 32)
    assert sa.sigattn_bwd_workspace_size(2, 2, 64, 64) == 2 * 512
    assert sa.sigattn_bwd_workspace_size(1, 1, 1, 96) == 0


def test_bad_arguments_rejected_before_any_device_work():
    lib = sa.library()
    null = None
    ws = ctypes.create_string_buffer(4096)
    # d = 96 is unsupported: status 2 whatever the pointers are
    assert lib.sigattn_fwd(null, null, null, null, null, 1, 1, 64, 96, null, 0, null) == 2
    # null lengths / workspace: invalid argument
    assert lib.sigattn_fwd(null, null, null, null, null, 1, 1, 64, 64, null, 0, null) == 1
    assert lib.sigattn_bwd_dq(null, null, null, null, null, null, 1, 1, 64, 64, null, 0, null) == 1
    assert lib.sigattn_bwd_dkdv(null, null, null, null, null, null, null, 1, 1, 64, 64, null, 0, null) == 1
    assert lib.sigattn_bwd(null, null, null, null, null, null, null, null, 1, 1, 64, 64, null, 0, null) == 1
    assert lib.sigattn_bwd(null, null, null, null, null, null, null, null, 1, 1, 64, 96, null, 0, null) == 2
    assert lib.sigattn_bwd_varlen(null, null, null, null, null, null, null, null, 1, 1, 64, 64, 64, null, 0,
                                  null) == 1
    # workspace too small
    lens = (ctypes.c_int * 1)(64)
    assert lib.sigattn_fwd(null, null, null, null, lens, 1, 1, 64, 64, ws, 16, null) == 1
    # enough for one work list but not for the whole-backward call's two
    one = sa.sigattn_workspace_size(1, 1, 64, 64)
    assert one < sa.sigattn_bwd_workspace_size(1, 1, 64, 64)
    assert lib.sigattn_bwd(null, null, null, null, null, null, null, lens, 1, 1, 64, 64, ws, one, null) == 1
    # negative sizes
    assert lib.sigattn_fwd(null, null, null, null, lens, -1, 1, 64, 64, ws, 4096, null) == 1
    assert lib.sigattn_plan(lens, 1, 1, 64, 64, 7, ws, 4096, null) == 1
    # packed layout: null cu_seqlens, unsupported d, total < 1, too many tokens
    for fn, nptr in ((lib.sigattn_fwd_varlen, 4), (lib.sigattn_bwd_dq_varlen, 5), (lib.sigattn_bwd_dkdv_varlen, 6)):
        ptrs = [null] * nptr
        assert fn(*ptrs, null, 1, 1, 64, 64, 64, null, 0, null) == 1
        assert fn(*ptrs, lens, 1, 1, 64, 64, 96, ws, 4096, null) == 2


@pytest.mark.parametrize("kind", [0, 1, 2])
def test_host_plan_matches_oracle_tiles(kind):
    rows = sa.sigattn_block_rows(kind)
    H, L = 3, 1000
    lens = np.array([0, 1, 127, 128, 129, 255, 256, 257, 999, 1000, 513, 640], dtype=np.int32)
    items = sa.sigattn_plan_host(lens, H, L, kind).numpy()
    got = sorted((int(bh) // H, int(bh) % H, int(m)) for bh, m in items)
    expect = [tuple(t) for t in oracle.tiles(lens, H, L, rows).tolist()]
    assert got == expect  # same set, each item once
    # longest sequence first (stable in batch order), heads then blocks ascending
    seq = [int(bh) // H for bh, _ in items]
    order = sorted(range(len(lens)), key=lambda b: (-lens[b], b))
    expect_seq = [b for b in order for _ in range(H * ((lens[b] + rows - 1) // rows))]
    assert seq == expect_seq


def test_host_plan_treats_out_of_range_lengths_as_empty():
    items = sa.sigattn_plan_host([5, -3, 70], 1, 64, 1).numpy()
    assert sorted(int(bh) for bh, _ in items) == [0]


def test_binding_rejects_cpu_tensors():
    q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        sa.sigattn_fwd(q, q, q, q, torch.zeros(1, dtype=torch.int32), torch.zeros(512, dtype=torch.uint8))
