"""fp64 CPU oracle for sigmoid attention -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package. The CUDA library never does, and nothing here imports
the CUDA library: the two share no code.

The arithmetic lives in ``sigattn_oracle.c`` (plain C, fp64, OpenMP over rows);
this module only compiles it with gcc, loads it with ctypes and converts arrays.
Every value it returns is computed in fp64 from the exact values of the inputs
(bf16 inputs upcast to fp64 lose nothing).

Source followed: "Better Models, Faster Training: Sigmoid Attention for
single-cell Foundation Models" -- sec. 2A (SigmoidAttn equation, bias
b = -log(n)), sec. 2B (sigma' = sigma(1 - sigma), bounded by 0.25; diagonal
Jacobian), sec. 2C (padding skipped on both sides; dQ and dK/dV gradients),
sec. 4A (the softmax comparison; softmax_forward states softmax attention over
the valid keys, as "Transformer Attention機構の効率化と最新派生モデル" writes it
in its "Vanilla Self-Attention" pseudo code example).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sigattn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP, -O2, no host-specific ISA flags)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", _SRC, "-o", _LIB, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.oracle_sigmoid.restype = ctypes.c_double
        lib.oracle_sigmoid.argtypes = [ctypes.c_double]
        lib.oracle_weight.restype = ctypes.c_double
        lib.oracle_weight.argtypes = [_dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        lib.oracle_fwd.restype = None
        lib.oracle_fwd.argtypes = [_dp, _dp, _dp, _dp, _ip] + [ctypes.c_int] * 4
        lib.oracle_bwd.restype = None
        lib.oracle_bwd.argtypes = [_dp] * 7 + [_ip] + [ctypes.c_int] * 4
        lib.oracle_rows.restype = None
        lib.oracle_rows.argtypes = [_dp] * 4 + [_ip] + [ctypes.c_int] * 5 + [_ip, _ip, ctypes.c_int, _dp]
        lib.oracle_softmax_fwd.restype = None
        lib.oracle_softmax_fwd.argtypes = [_dp] * 5 + [_ip] + [ctypes.c_int] * 4
        lib.oracle_tiles.restype = ctypes.c_int
        lib.oracle_tiles.argtypes = [_ip] + [ctypes.c_int] * 4 + [_ip, ctypes.c_int]
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact fp64 copy of an array-like (torch tensors of any float dtype included)."""
    if hasattr(x, "detach"):  # torch tensor: bf16 -> fp32 -> fp64 is exact
        import torch

        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _ptr(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def sigmoid(x: float) -> float:
    return _load().oracle_sigmoid(float(x))


def forward(q, k, v, lengths) -> np.ndarray:
    """O for padded [B,H,L,d] inputs (rows i >= n_b are 0)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    lens = _i32(lengths)
    B, H, L, d = q.shape
    o = np.zeros_like(q)
    _load().oracle_fwd(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), _ptr(o, _dp), _ptr(lens, _ip), B, H, L, d)
    return o


def backward(q, k, v, dout, lengths):
    """(dQ, dK, dV) for padded [B,H,L,d] inputs and upstream gradient dO."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    lens = _i32(lengths)
    B, H, L, d = q.shape
    dq, dk, dv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    _load().oracle_bwd(*[_ptr(a, _dp) for a in (q, k, v, dout, dq, dk, dv)], _ptr(lens, _ip), B, H, L, d)
    return dq, dk, dv


def softmax_forward(q, k, v, lengths):
    """The softmax counterpart: (O [B,H,L,d], lse [B,H,L]) over the valid keys,
    rows i >= n_b zero (see oracle_softmax_fwd_row)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    lens = _i32(lengths)
    B, H, L, d = q.shape
    o = np.zeros_like(q)
    lse = np.zeros((B, H, L), dtype=np.float64)
    _load().oracle_softmax_fwd(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), _ptr(o, _dp), _ptr(lse, _dp),
                               _ptr(lens, _ip), B, H, L, d)
    return o, lse


ROW_KIND = {"o": 0, "dq": 1, "dk": 2, "dv": 3}


def rows(which: str, q, k, v, dout, lengths, bh, row) -> np.ndarray:
    """Selected output rows: out[s] = <which>[bh[s] // H, bh[s] % H, row[s], :]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    dout = _f64(dout) if dout is not None else np.zeros_like(q)
    lens = _i32(lengths)
    B, H, L, d = q.shape
    if d > 512:
        raise ValueError("oracle.rows supports d <= 512")
    bh = _i32(bh)
    row = _i32(row)
    out = np.zeros((len(bh), d), dtype=np.float64)
    _load().oracle_rows(*[_ptr(a, _dp) for a in (q, k, v, dout)], _ptr(lens, _ip), B, H, L, d,
                        ROW_KIND[which], _ptr(bh, _ip), _ptr(row, _ip), len(bh), _ptr(out, _dp))
    return out


def weight(q_slice, k_slice, n: int, i: int, j: int) -> float:
    """P_ij of one (b,h) slice given as [L,d] arrays."""
    q, k = _f64(q_slice), _f64(k_slice)
    return _load().oracle_weight(_ptr(q, _dp), _ptr(k, _dp), int(n), q.shape[1], int(i), int(j))


def tiles(lengths, H: int, L: int, block: int) -> np.ndarray:
    """Active work items (b, h, m) in canonical order, as an int32 array [count, 3]."""
    lens = _i32(lengths)
    B = len(lens)
    lib = _load()
    count = lib.oracle_tiles(_ptr(lens, _ip), B, H, L, block, None, 0)
    out = np.zeros((max(count, 1), 3), dtype=np.int32)
    lib.oracle_tiles(_ptr(lens, _ip), B, H, L, block, _ptr(out, _ip), count)
    return out[:count]
