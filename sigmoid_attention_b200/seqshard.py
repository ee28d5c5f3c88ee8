"""Sequence-sharded sigmoid attention: one process per GPU, keys split by position.

Every rank holds all query rows (Q and dO, [B, H, Lmax, d]) and one contiguous
range of key rows (K and V, [B, H, count, d]) of every sequence. Each weight
sigma(q.k / sqrt(d) - ln n) is computed on its own, with no normalisation
over the keys ("Better Models, Faster Training: Sigmoid Attention for
single-cell Foundation Models", sec. 2A), so

  * O is the plain sum over ranks of each rank's fp32 partial output over its
    keys: one all-reduce, no log-sum-exp merge;
  * dQ = scale * dS K is summed the same way;
  * dK and dV of a rank's keys need all queries and dO only, which every rank
    has, so they need no exchange at all.

The kernels are the library's key-range calls (sigattn_fwd_partial,
sigattn_bwd_dq_partial, sigattn_bwd_dkdv_range, sigattn_cast_bf16); the sum is
torch.distributed.all_reduce (NCCL on GPUs: plain device buffers, no
multicast). This module only orders those calls.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (make_workspace, sigattn_bwd_dkdv_range, sigattn_bwd_dq_partial, sigattn_cast_bf16,
               sigattn_fwd_partial)

ALIGN = 128  # range boundaries on whole 128-row blocks keep dK/dV bit-identical to the unsharded call


def key_range(rank: int, world: int, Lmax: int, align: int = ALIGN) -> tuple[int, int]:
    """(begin, count) of the keys rank `rank` of `world` holds: consecutive
    ranges of equal length (a multiple of `align`) tiling [0, Lmax); the last
    may be shorter and trailing ranks may be empty (count 0)."""
    if world < 1 or not 0 <= rank < world or Lmax < 1:
        raise ValueError("need world >= 1, 0 <= rank < world and Lmax >= 1")
    per = -(-Lmax // world)
    per = -(-per // align) * align
    begin = min(rank * per, Lmax)
    return begin, min(per, Lmax - begin)


def merge_partials_(partial: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the ranks' partial outputs in place (all-reduce); returns `partial`."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
    return partial


def _to_bf16(x32: torch.Tensor) -> torch.Tensor:
    y = torch.empty(x32.shape, dtype=torch.bfloat16, device=x32.device)
    sigattn_cast_bf16(x32, y)
    return y


def forward(q, k_local, v_local, lengths, key_begin: int, group=None, workspace=None) -> torch.Tensor:
    """O (bf16 [B, H, Lmax, d]) of all queries, from this rank's keys
    [key_begin, key_begin + k_local.shape[2]) and the other ranks' partials."""
    B, H, L, d = q.shape
    if workspace is None:
        workspace = make_workspace(B, H, L, d, q.device)
    if k_local.shape[2] > 0:  # the call writes every element (zeros where no key of the range applies)
        o32 = torch.empty((B, H, L, d), dtype=torch.float32, device=q.device)
        sigattn_fwd_partial(q, k_local, v_local, o32, lengths, key_begin, workspace)
    else:  # a rank without keys contributes nothing
        o32 = torch.zeros((B, H, L, d), dtype=torch.float32, device=q.device)
    return _to_bf16(merge_partials_(o32, group))


def backward(q, k_local, v_local, dout, lengths, key_begin: int, group=None, workspace=None):
    """(dQ of all queries, bf16, summed over ranks; dK and dV of this rank's keys)."""
    B, H, L, d = q.shape
    if workspace is None:
        workspace = make_workspace(B, H, L, d, q.device)
    dk, dv = torch.empty_like(k_local), torch.empty_like(v_local)
    if k_local.shape[2] > 0:
        dq32 = torch.empty((B, H, L, d), dtype=torch.float32, device=q.device)
        sigattn_bwd_dq_partial(q, k_local, v_local, dout, dq32, lengths, key_begin, workspace)
        sigattn_bwd_dkdv_range(q, k_local, v_local, dout, dk, dv, lengths, key_begin, workspace)
    else:
        dq32 = torch.zeros((B, H, L, d), dtype=torch.float32, device=q.device)
    return _to_bf16(merge_partials_(dq32, group)), dk, dv


class SeqShardedSigmoidAttention(torch.autograd.Function):
    """Autograd wrapper: q (all rows, replicated on every rank), this rank's
    k and v key range; returns the full O. The gradient of q is the summed dQ
    (identical on every rank); k and v get their own range's gradients."""

    @staticmethod
    def forward(ctx, q, k_local, v_local, lengths, key_begin, group=None):
        q, k_local, v_local = q.contiguous(), k_local.contiguous(), v_local.contiguous()
        ws = make_workspace(*q.shape, q.device)
        o = forward(q, k_local, v_local, lengths, key_begin, group, ws)
        ctx.save_for_backward(q, k_local, v_local, lengths, ws)
        ctx.key_begin, ctx.group = key_begin, group
        return o

    @staticmethod
    def backward(ctx, do):
        q, k_local, v_local, lengths, ws = ctx.saved_tensors
        dq, dk, dv = backward(q, k_local, v_local, do.contiguous(), lengths, ctx.key_begin, ctx.group, ws)
        return dq, dk, dv, None, None, None


def sharded_sigmoid_attention(q, k_local, v_local, lengths, key_begin: int, group=None) -> torch.Tensor:
    return SeqShardedSigmoidAttention.apply(q, k_local, v_local, lengths, int(key_begin), group)
