"""Python binding of the B200 sigmoid-attention C ABI (``include/sigattn.h``).

Argument marshalling only: each ``sigattn_*`` function here passes device
pointers, sizes and the current CUDA stream to the function of the same name
in ``libsigattn.so``; every step of the computation runs in the library's CUDA
kernels. PyTorch provides device memory and streams. There is no fallback: if
the library is missing or a call fails, an exception is raised.

The library computes O = sigma(Q K^T / sqrt(d) - ln n) V over padded
[B, H, Lmax, d] bf16 batches with per-sequence valid lengths n, and the
gradients dQ, dK, dV ("Better Models, Faster Training: Sigmoid Attention for
single-cell Foundation Models", sec. 2A-2C).
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "SigattnError", "library", "library_path", "sigattn_version", "sigattn_status_str", "sigattn_block_rows",
    "sigattn_workspace_size", "sigattn_bwd_workspace_size", "sigattn_fwd", "sigattn_fwd_noalloc", "sigattn_bwd",
    "sigattn_bwd_dq", "sigattn_bwd_dkdv", "sigattn_plan",
    "sigattn_plan_host", "sigattn_read_error", "sigattn_last_error", "sigattn_eval_sigmoid", "read_plan", "sigattn_selftest_wait_timeout", "make_workspace", "forward", "backward",
    "sigattn_fwd_varlen", "sigattn_bwd_varlen", "sigattn_bwd_dq_varlen", "sigattn_bwd_dkdv_varlen",
    "sigattn_fwd_partial", "sigattn_bwd_dq_partial", "sigattn_bwd_dkdv_range", "sigattn_cast_bf16",
    "sigattn_softmax_fwd",
    "KIND_FWD", "KIND_DQ", "KIND_DKDV", "SigmoidAttentionFunction", "sigmoid_attention",
    "SigmoidAttentionVarlenFunction", "sigmoid_attention_varlen",
]

KIND_FWD, KIND_DQ, KIND_DKDV = 0, 1, 2
STATUS = {0: "SIGATTN_OK", 1: "SIGATTN_ERR_INVALID_ARG", 2: "SIGATTN_ERR_UNSUPPORTED", 3: "SIGATTN_ERR_CUDA",
          4: "SIGATTN_ERR_TIMEOUT"}

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsigattn.so")
_lib = None

_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t


class SigattnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")


def library_path() -> str:
    return _LIB_PATH


def library():
    """Load ``libsigattn.so`` (built in-tree by ``sigmoid_attention_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: run `python -m sigmoid_attention_b200.build` first")
        lib = ctypes.CDLL(_LIB_PATH)
        lib.sigattn_version.restype = _i
        lib.sigattn_version.argtypes = []
        lib.sigattn_status_str.restype = ctypes.c_char_p
        lib.sigattn_status_str.argtypes = [_i]
        lib.sigattn_block_rows.restype = _i
        lib.sigattn_block_rows.argtypes = [_i]
        lib.sigattn_workspace_size.restype = _sz
        lib.sigattn_workspace_size.argtypes = [_i] * 4
        lib.sigattn_fwd.restype = _i
        lib.sigattn_fwd.argtypes = [_vp] * 5 + [_i] * 4 + [_vp, _sz, _vp]
        lib.sigattn_bwd_dq.restype = _i
        lib.sigattn_bwd_dq.argtypes = [_vp] * 6 + [_i] * 4 + [_vp, _sz, _vp]
        lib.sigattn_bwd_dkdv.restype = _i
        lib.sigattn_bwd_dkdv.argtypes = [_vp] * 7 + [_i] * 4 + [_vp, _sz, _vp]
        lib.sigattn_bwd_workspace_size.restype = _sz
        lib.sigattn_bwd_workspace_size.argtypes = [_i] * 4
        lib.sigattn_bwd.restype = _i
        lib.sigattn_bwd.argtypes = [_vp] * 8 + [_i] * 4 + [_vp, _sz, _vp]
        lib.sigattn_fwd_varlen.restype = _i
        lib.sigattn_fwd_varlen.argtypes = [_vp] * 5 + [_i] * 5 + [_vp, _sz, _vp]
        lib.sigattn_bwd_dq_varlen.restype = _i
        lib.sigattn_bwd_dq_varlen.argtypes = [_vp] * 6 + [_i] * 5 + [_vp, _sz, _vp]
        lib.sigattn_bwd_dkdv_varlen.restype = _i
        lib.sigattn_bwd_dkdv_varlen.argtypes = [_vp] * 7 + [_i] * 5 + [_vp, _sz, _vp]
        lib.sigattn_bwd_varlen.restype = _i
        lib.sigattn_bwd_varlen.argtypes = [_vp] * 8 + [_i] * 5 + [_vp, _sz, _vp]
        lib.sigattn_plan.restype = _i
        lib.sigattn_plan.argtypes = [_vp] + [_i] * 5 + [_vp, _sz, _vp]
        lib.sigattn_plan_host.restype = _i
        lib.sigattn_plan_host.argtypes = [_vp] + [_i] * 4 + [_vp, _i, ctypes.POINTER(_i)]
        lib.sigattn_fwd_noalloc.restype = _i
        lib.sigattn_fwd_noalloc.argtypes = [_vp] * 5 + [_i] * 4 + [_vp, _vp]
        lib.sigattn_selftest_wait_timeout.restype = _i
        lib.sigattn_selftest_wait_timeout.argtypes = [_vp, _sz, _i, _vp]
        lib.sigattn_last_error.restype = ctypes.c_char_p
        lib.sigattn_last_error.argtypes = []
        lib.sigattn_fwd_partial.restype = _i
        lib.sigattn_fwd_partial.argtypes = [_vp] * 5 + [_i] * 6 + [_vp, _sz, _vp]
        lib.sigattn_bwd_dq_partial.restype = _i
        lib.sigattn_bwd_dq_partial.argtypes = [_vp] * 6 + [_i] * 6 + [_vp, _sz, _vp]
        lib.sigattn_bwd_dkdv_range.restype = _i
        lib.sigattn_bwd_dkdv_range.argtypes = [_vp] * 7 + [_i] * 6 + [_vp, _sz, _vp]
        lib.sigattn_softmax_fwd.restype = _i
        lib.sigattn_softmax_fwd.argtypes = [_vp] * 5 + [_i] * 4 + [_vp, _sz, _vp]
        lib.sigattn_cast_bf16.restype = _i
        lib.sigattn_cast_bf16.argtypes = [_vp, _vp, ctypes.c_longlong, _vp]
        lib.sigattn_eval_sigmoid.restype = _i
        lib.sigattn_eval_sigmoid.argtypes = [_vp, _vp, _vp, _i, _i, _i, _vp]
        lib.sigattn_read_error.restype = _i
        lib.sigattn_read_error.argtypes = [_vp, ctypes.POINTER(_i), _vp]
        _lib = lib
    return _lib


def _check(fn: str, status: int) -> None:
    if status != 0:
        err = SigattnError(fn, status)
        if status in (2, 3):
            err.args = (f"{err.args[0]} ({library().sigattn_last_error().decode()})",)
        raise err


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _dims(q: torch.Tensor):
    if q.dim() != 4:
        raise ValueError("expected a [B, H, Lmax, d] tensor")
    return tuple(int(x) for x in q.shape)


def _dev(t: torch.Tensor, name: str, dtype=torch.bfloat16) -> int:
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")
    return t.data_ptr()


def sigattn_version() -> int:
    return library().sigattn_version()


def sigattn_status_str(status: int) -> str:
    return library().sigattn_status_str(status).decode()


def sigattn_block_rows(kind: int) -> int:
    return library().sigattn_block_rows(kind)


def sigattn_workspace_size(B: int, H: int, Lmax: int, d: int) -> int:
    return library().sigattn_workspace_size(B, H, Lmax, d)


def sigattn_bwd_workspace_size(B: int, H: int, Lmax: int, d: int) -> int:
    return library().sigattn_bwd_workspace_size(B, H, Lmax, d)


def make_workspace(B: int, H: int, Lmax: int, d: int, device=None) -> torch.Tensor:
    """A zero-initialised workspace (uint8 CUDA tensor) big enough for any
    call, ``sigattn_bwd`` (two work lists) included."""
    n = max(sigattn_workspace_size(B, H, Lmax, d), sigattn_bwd_workspace_size(B, H, Lmax, d))
    if n == 0:
        raise SigattnError("sigattn_workspace_size", 2)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def sigattn_fwd(q, k, v, o, lengths, workspace, stream=None) -> None:
    B, H, L, d = _dims(q)
    _check("sigattn_fwd", library().sigattn_fwd(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(lengths, "lengths", torch.int32),
        B, H, L, d, _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream_ptr(stream)))


def sigattn_softmax_fwd(q, k, v, o, lengths, workspace, stream=None) -> None:
    """The softmax counterpart of sigattn_fwd (d = 64, forward only)."""
    B, H, L, d = _dims(q)
    _check("sigattn_softmax_fwd", library().sigattn_softmax_fwd(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(lengths, "lengths", torch.int32),
        B, H, L, d, _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream_ptr(stream)))


def sigattn_fwd_noalloc(q, k, v, o, lengths, status_out=None, stream=None) -> None:
    """Forward pass without a workspace, for callers that cannot allocate
    device memory: the library's own fixed scratch array is used instead."""
    B, H, L, d = _dims(q)
    st_ptr = _dev(status_out, "status_out", torch.int32) if status_out is not None else None
    _check("sigattn_fwd_noalloc", library().sigattn_fwd_noalloc(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(lengths, "lengths", torch.int32),
        B, H, L, d, st_ptr, _stream_ptr(stream)))


def sigattn_bwd_dq(q, k, v, dout, dq, lengths, workspace, stream=None) -> None:
    B, H, L, d = _dims(q)
    _check("sigattn_bwd_dq", library().sigattn_bwd_dq(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(dout, "dout"), _dev(dq, "dq"),
        _dev(lengths, "lengths", torch.int32), B, H, L, d, _dev(workspace, "workspace", torch.uint8),
        workspace.numel(), _stream_ptr(stream)))


def sigattn_bwd_dkdv(q, k, v, dout, dk, dv, lengths, workspace, stream=None) -> None:
    B, H, L, d = _dims(q)
    _check("sigattn_bwd_dkdv", library().sigattn_bwd_dkdv(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(dout, "dout"), _dev(dk, "dk"), _dev(dv, "dv"),
        _dev(lengths, "lengths", torch.int32), B, H, L, d, _dev(workspace, "workspace", torch.uint8),
        workspace.numel(), _stream_ptr(stream)))


def sigattn_bwd(q, k, v, dout, dq, dk, dv, lengths, workspace, stream=None) -> None:
    """dQ, dK and dV in one call (the two backward kernels overlapped; results
    identical to sigattn_bwd_dq + sigattn_bwd_dkdv)."""
    B, H, L, d = _dims(q)
    _check("sigattn_bwd", library().sigattn_bwd(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(dout, "dout"), _dev(dq, "dq"), _dev(dk, "dk"),
        _dev(dv, "dv"), _dev(lengths, "lengths", torch.int32), B, H, L, d,
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream_ptr(stream)))


def sigattn_fwd_partial(q, k, v, o_partial, lengths, key_begin: int, workspace, stream=None) -> None:
    """Key-range forward: k, v are [B, H, key_count, d] bf16 holding keys
    key_begin .. key_begin + key_count - 1 of every sequence; o_partial is the
    fp32 [B, H, Lmax, d] contribution of those keys (see the C header)."""
    B, H, L, d = _dims(q)
    _check("sigattn_fwd_partial", library().sigattn_fwd_partial(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o_partial, "o_partial", torch.float32),
        _dev(lengths, "lengths", torch.int32), B, H, L, d, int(key_begin), int(k.shape[2]),
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream_ptr(stream)))


def sigattn_bwd_dq_partial(q, k, v, dout, dq_partial, lengths, key_begin: int, workspace, stream=None) -> None:
    B, H, L, d = _dims(q)
    _check("sigattn_bwd_dq_partial", library().sigattn_bwd_dq_partial(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(dout, "dout"), _dev(dq_partial, "dq_partial", torch.float32),
        _dev(lengths, "lengths", torch.int32), B, H, L, d, int(key_begin), int(k.shape[2]),
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream_ptr(stream)))


def sigattn_bwd_dkdv_range(q, k, v, dout, dk, dv, lengths, key_begin: int, workspace, stream=None) -> None:
    B, H, L, d = _dims(q)
    _check("sigattn_bwd_dkdv_range", library().sigattn_bwd_dkdv_range(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(dout, "dout"), _dev(dk, "dk"), _dev(dv, "dv"),
        _dev(lengths, "lengths", torch.int32), B, H, L, d, int(key_begin), int(k.shape[2]),
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream_ptr(stream)))


def sigattn_cast_bf16(x, y, stream=None) -> None:
    """y (bf16) = x (fp32) rounded to nearest even; same number of elements."""
    if x.numel() != y.numel():
        raise ValueError("x and y must have the same number of elements")
    _check("sigattn_cast_bf16", library().sigattn_cast_bf16(
        _dev(x, "x", torch.float32), _dev(y, "y"), x.numel(), _stream_ptr(stream)))


def _packed_dims(q: torch.Tensor):
    if q.dim() != 3:
        raise ValueError("expected a packed [total, H, d] tensor")
    return tuple(int(x) for x in q.shape)


def sigattn_fwd_varlen(q, k, v, o, cu_seqlens, max_seqlen: int, workspace, stream=None) -> None:
    """Packed layout: q, k, v, o are [total, H, d]; cu_seqlens is int32 [B + 1]."""
    total, H, d = _packed_dims(q)
    B = cu_seqlens.numel() - 1
    _check("sigattn_fwd_varlen", library().sigattn_fwd_varlen(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(o, "o"), _dev(cu_seqlens, "cu_seqlens", torch.int32),
        B, H, int(max_seqlen), total, d, _dev(workspace, "workspace", torch.uint8), workspace.numel(),
        _stream_ptr(stream)))


def sigattn_bwd_dq_varlen(q, k, v, dout, dq, cu_seqlens, max_seqlen: int, workspace, stream=None) -> None:
    total, H, d = _packed_dims(q)
    B = cu_seqlens.numel() - 1
    _check("sigattn_bwd_dq_varlen", library().sigattn_bwd_dq_varlen(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(dout, "dout"), _dev(dq, "dq"),
        _dev(cu_seqlens, "cu_seqlens", torch.int32), B, H, int(max_seqlen), total, d,
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream_ptr(stream)))


def sigattn_bwd_varlen(q, k, v, dout, dq, dk, dv, cu_seqlens, max_seqlen: int, workspace, stream=None) -> None:
    """Packed-layout counterpart of sigattn_bwd."""
    total, H, d = _packed_dims(q)
    B = cu_seqlens.numel() - 1
    _check("sigattn_bwd_varlen", library().sigattn_bwd_varlen(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(dout, "dout"), _dev(dq, "dq"), _dev(dk, "dk"),
        _dev(dv, "dv"), _dev(cu_seqlens, "cu_seqlens", torch.int32), B, H, int(max_seqlen), total, d,
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream_ptr(stream)))


def sigattn_bwd_dkdv_varlen(q, k, v, dout, dk, dv, cu_seqlens, max_seqlen: int, workspace, stream=None) -> None:
    total, H, d = _packed_dims(q)
    B = cu_seqlens.numel() - 1
    _check("sigattn_bwd_dkdv_varlen", library().sigattn_bwd_dkdv_varlen(
        _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(dout, "dout"), _dev(dk, "dk"), _dev(dv, "dv"),
        _dev(cu_seqlens, "cu_seqlens", torch.int32), B, H, int(max_seqlen), total, d,
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), _stream_ptr(stream)))


def sigattn_plan(lengths, B, H, Lmax, d, kind, workspace, stream=None) -> None:
    _check("sigattn_plan", library().sigattn_plan(
        _dev(lengths, "lengths", torch.int32), B, H, Lmax, d, kind, _dev(workspace, "workspace", torch.uint8),
        workspace.numel(), _stream_ptr(stream)))


def read_plan(workspace: torch.Tensor) -> torch.Tensor:
    """The (bh, block) pairs the last plan wrote, as an int32 CPU tensor [count, 2]."""
    words = workspace.view(torch.int32).cpu()
    count = int(words[2])
    return words[64:64 + 4 * count].view(count, 4)[:, :2].clone()


def sigattn_plan_host(lengths, H: int, Lmax: int, kind: int) -> torch.Tensor:
    """Host statement of the schedule: int32 [count, 2] of (bh, block) pairs."""
    lens = torch.as_tensor(lengths, dtype=torch.int32).contiguous()
    B = lens.numel()
    count = ctypes.c_int(0)
    lib = library()
    _check("sigattn_plan_host", lib.sigattn_plan_host(lens.data_ptr(), B, H, Lmax, kind, None, 0,
                                                      ctypes.byref(count)))
    out = torch.zeros(max(count.value, 1), 2, dtype=torch.int32)
    _check("sigattn_plan_host", lib.sigattn_plan_host(lens.data_ptr(), B, H, Lmax, kind, out.data_ptr(),
                                                      count.value, ctypes.byref(count)))
    return out[:count.value]


def sigattn_selftest_wait_timeout(workspace, limit_us: int = 20000, stream=None) -> None:
    """Enqueue the diagnostic kernel whose bounded wait must expire (see the header)."""
    _check("sigattn_selftest_wait_timeout", library().sigattn_selftest_wait_timeout(
        _dev(workspace, "workspace", torch.uint8), workspace.numel(), int(limit_us), _stream_ptr(stream)))


def sigattn_eval_sigmoid(scores, d: int, n: int, stream=None):
    """(P, slope) of float32 CUDA scores as the kernels compute them:
    P = sigma(s / sqrt(d) - ln n), slope = P (1 - P)."""
    p, slope = torch.empty_like(scores), torch.empty_like(scores)
    _check("sigattn_eval_sigmoid", library().sigattn_eval_sigmoid(
        _dev(scores, "scores", torch.float32), _dev(p, "p", torch.float32), _dev(slope, "slope", torch.float32),
        scores.numel(), int(d), int(n), _stream_ptr(stream)))
    return p, slope


def sigattn_last_error() -> str:
    return library().sigattn_last_error().decode()


def sigattn_read_error(workspace, stream=None):
    """Synchronise, read and clear the workspace's sticky error word: (status, site)."""
    site = ctypes.c_int(0)
    st = library().sigattn_read_error(_dev(workspace, "workspace", torch.uint8), ctypes.byref(site),
                                      _stream_ptr(stream))
    return st, site.value


# ---------------------------------------------------------------------------
# Convenience wrappers (allocate outputs with torch, then call the C ABI)
# ---------------------------------------------------------------------------
def forward(q, k, v, lengths, workspace=None, stream=None) -> torch.Tensor:
    B, H, L, d = _dims(q)
    if workspace is None:
        workspace = make_workspace(B, H, L, d, q.device)
    o = torch.empty_like(q)
    sigattn_fwd(q, k, v, o, lengths, workspace, stream)
    return o


def backward(q, k, v, dout, lengths, workspace=None, stream=None):
    B, H, L, d = _dims(q)
    if workspace is None:
        workspace = make_workspace(B, H, L, d, q.device)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    sigattn_bwd(q, k, v, dout, dq, dk, dv, lengths, workspace, stream)
    return dq, dk, dv


def _check_device_status(fn: str, workspace, check: bool) -> None:
    """With ``check`` (or SIGATTN_CHECK=1 in the environment), synchronise and
    raise if a kernel flagged an out-of-range length or an expired wait in the
    workspace's sticky status word (otherwise such a sequence's outputs are
    zeros and nothing is raised)."""
    if not (check or os.environ.get("SIGATTN_CHECK", "0") == "1"):
        return
    st, site = sigattn_read_error(workspace)
    if st != 0:
        err = SigattnError(fn, st)
        err.args = (f"{err.args[0]} (device status, site {site})",)
        raise err


class SigmoidAttentionFunction(torch.autograd.Function):
    """Autograd wrapper: forward with ``sigattn_fwd``, backward with
    ``sigattn_bwd`` (dQ, dK and dV in one call; a drop-in for softmax
    attention over padded batches)."""

    @staticmethod
    def forward(ctx, q, k, v, lengths, check=False):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        ws = make_workspace(*_dims(q), q.device)
        o = forward(q, k, v, lengths, ws)
        _check_device_status("sigattn_fwd", ws, check)
        ctx.save_for_backward(q, k, v, lengths, ws)
        ctx.check = check
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, lengths, ws = ctx.saved_tensors
        dq, dk, dv = backward(q, k, v, do.contiguous(), lengths, ws)
        _check_device_status("sigattn_bwd", ws, ctx.check)
        return dq, dk, dv, None, None


def sigmoid_attention(q, k, v, lengths, check: bool = False) -> torch.Tensor:
    """O = sigma(q k^T / sqrt(d) - ln n) v over padded [B, H, Lmax, d] bf16
    tensors, differentiable in q, k, v. ``check=True`` synchronises after the
    forward and the backward calls and raises SigattnError when a kernel
    reported a problem (an out-of-range length, an expired wait)."""
    return SigmoidAttentionFunction.apply(q, k, v, lengths, check)


class SigmoidAttentionVarlenFunction(torch.autograd.Function):
    """Autograd wrapper of the packed-layout calls: q, k, v are [total, H, d]
    with sequences back to back as given by cu_seqlens (int32 [B + 1])."""

    @staticmethod
    def forward(ctx, q, k, v, cu_seqlens, max_seqlen, check=False):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        _, H, d = _packed_dims(q)
        ws = make_workspace(cu_seqlens.numel() - 1, H, max_seqlen, d, q.device)
        o = torch.empty_like(q)
        sigattn_fwd_varlen(q, k, v, o, cu_seqlens, max_seqlen, ws)
        _check_device_status("sigattn_fwd_varlen", ws, check)
        ctx.save_for_backward(q, k, v, cu_seqlens, ws)
        ctx.max_seqlen = max_seqlen
        ctx.check = check
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, cu_seqlens, ws = ctx.saved_tensors
        do = do.contiguous()
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        sigattn_bwd_varlen(q, k, v, do, dq, dk, dv, cu_seqlens, ctx.max_seqlen, ws)
        _check_device_status("sigattn_bwd_varlen", ws, ctx.check)
        return dq, dk, dv, None, None, None


def sigmoid_attention_varlen(q, k, v, cu_seqlens, max_seqlen: int, check: bool = False) -> torch.Tensor:
    """The packed-layout counterpart of ``sigmoid_attention`` ([total, H, d]
    tensors, int32 cu_seqlens [B + 1]); ``check`` as there."""
    return SigmoidAttentionVarlenFunction.apply(q, k, v, cu_seqlens, int(max_seqlen), check)
