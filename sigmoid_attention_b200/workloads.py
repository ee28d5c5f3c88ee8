"""Seeded synthetic workloads for sigmoid attention (shared by tests and bench).

This module holds no attention arithmetic: it only draws inputs. Both the CUDA
library and the fp64 oracle are fed from here, so neither side generates its
own data.

Workloads stand in for padded batches of single-cell expression profiles, where
each cell has from hundreds to thousands of expressed genes and cells are padded
to the batch maximum ("Better Models, Faster Training: Sigmoid Attention for
single-cell Foundation Models", sec. 1). The shapes are the five benchmark cases
of this library: a tiny correctness case, a scRNA-seq-shaped ragged batch, a
dense unpadded d=128 case, an 8K long-context case and a padding sweep.

Recipe: Q, K, V, dO are i.i.d. N(0,1) drawn as fp32 by a CPU
``torch.Generator`` seeded with ``seed`` (in that order: q, k, v, dout), then
rounded to bf16. Padded rows hold N(0,1) values too (they must be ignored).
Lengths come from ``numpy.random.default_rng(seed)``.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    L: int  # padded length Lmax
    d: int
    seed: int
    lengths_rule: str  # how lengths are drawn (documentation)

    def lengths(self) -> np.ndarray:
        return _draw_lengths(self)

    def fwd_flops(self, lengths=None) -> float:
        """Valid-pair forward FLOPs: 4*d per (i,j) with i,j < n_b (two matmuls)."""
        n = np.asarray(self.lengths() if lengths is None else lengths, dtype=np.float64)
        return 4.0 * self.d * self.H * float(np.sum(n * n))

    def bwd_flops(self, lengths=None) -> float:
        """Valid-pair backward FLOPs: 10*d per (i,j) (five matmuls, the usual count)."""
        n = np.asarray(self.lengths() if lengths is None else lengths, dtype=np.float64)
        return 10.0 * self.d * self.H * float(np.sum(n * n))

    def describe(self) -> dict:
        return {"workload": self.name, "B": self.B, "H": self.H, "Lmax": self.L, "d": self.d,
                "seed": self.seed, "lengths": self.lengths_rule}


def _sweep(p_index: int, pct: int) -> Workload:
    return Workload(f"pad_sweep_p{pct:02d}", 16, 12, 4096, 64, 1005 + p_index,
                    f"uniform with mean padding {pct}%")


WORKLOADS = {
    "tiny": Workload("tiny", 2, 2, 64, 64, 1001, "{37, 64}"),
    "scrna_ragged": Workload("scrna_ragged", 8, 8, 2048, 64, 1002, "uniform integers in [256, 2048]"),
    "dense_d128": Workload("dense_d128", 4, 16, 4096, 128, 1003, "all 4096"),
    "long_8k": Workload("long_8k", 2, 16, 8192, 64, 1004, "log-uniform in [1024, 8192]"),
    "pad_sweep_p00": _sweep(0, 0),
    "pad_sweep_p25": _sweep(1, 25),
    "pad_sweep_p50": _sweep(2, 50),
    "pad_sweep_p75": _sweep(3, 75),
}


def _draw_lengths(w: Workload) -> np.ndarray:
    rng = np.random.default_rng(w.seed)
    if w.name == "tiny":
        return np.array([37, 64], dtype=np.int32)
    if w.name == "scrna_ragged":
        return rng.integers(256, 2048 + 1, size=w.B).astype(np.int32)
    if w.name == "dense_d128":
        return np.full(w.B, w.L, dtype=np.int32)
    if w.name == "long_8k":
        u = rng.random(w.B)
        return np.clip(np.round(1024.0 * np.exp(u * math.log(8.0))), 1024, 8192).astype(np.int32)
    if w.name.startswith("pad_sweep_p"):
        # Uniform integers centred on m = (1 - p) * L, as wide as [1, L] allows,
        # so the mean padding is p.
        p = int(w.name[-2:]) / 100.0
        m = (1.0 - p) * w.L
        lo = int(max(1, round(2 * m - w.L)))
        hi = int(min(w.L, round(2 * m)))
        return rng.integers(lo, hi + 1, size=w.B).astype(np.int32)
    raise KeyError(w.name)


def make_inputs(B: int, H: int, L: int, d: int, seed: int, dtype=torch.bfloat16):
    """q, k, v, dout as CPU tensors [B,H,L,d], N(0,1) in fp32 rounded to ``dtype``."""
    g = torch.Generator().manual_seed(seed)
    out = []
    for _ in range(4):
        out.append(torch.randn((B, H, L, d), generator=g, dtype=torch.float32).to(dtype))
    return tuple(out)


def workload_inputs(w: Workload):
    """(q, k, v, dout, lengths) on the CPU for a named workload."""
    q, k, v, dout = make_inputs(w.B, w.H, w.L, w.d, w.seed)
    return q, k, v, dout, torch.from_numpy(w.lengths())


def random_lengths(B: int, L: int, seed: int, lo: int = 1) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return rng.integers(lo, L + 1, size=B).astype(np.int32)
