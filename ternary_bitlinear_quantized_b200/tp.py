"""Tensor parallelism of the BitNet FFN block over ranks (one process per GPU).

BitNetMLP.forward = down(ffn_sub_norm(act(gate(x)) * up(x))) ("Add optional RMSNorm support
to BitNet quantization", review thread) is split over the intermediate dimension I:

* gate/up: each rank holds a contiguous block of I / world weight ROWS of W_gate and W_up
  (an I2_S row block is a contiguous byte range; the tensor's one scale beta is the whole
  tensor's and every shard carries it in its trailer), so each rank produces the matching
  columns of h with ``bitnet_bitlinear_gate_up_act``;
* ffn_sub_norm: its reductions over the whole row of h are finished across ranks: max |h|
  (all-reduce MAX), the exact fixed-point sum of h^2 on the grid of the whole row
  (all-reduce SUM, int64), max |y| (all-reduce MAX); each rank then quantises its columns
  with the shared scale;
* down: each rank holds the same block of in-feature COLUMNS of W_down and computes its
  share of the int32 accumulators (``bitnet_bitlinear_acc`` with its shard's activation
  sum); the shares are summed over ranks (all-reduce SUM, int32) and dequantised once.

Every collective combines integers or maxima, so the result is bit-identical to the
single-GPU ``ffn_block``.  The x input is replicated (every rank quantises it itself).
The collectives default to ``torch.distributed`` (NCCL between GPUs); a caller may pass
its own reduction functions.  This module only marshals tensors and orders the calls:
the arithmetic runs in the library's kernels.
"""
from __future__ import annotations

import dataclasses

import torch

from . import (bitlinear_acc, bitlinear_gate_up_act, dequant_acc, i2s_packed_bytes, rmsnorm_quant_act,
               subnorm_shard_amax, subnorm_shard_quant, subnorm_shard_sumsq, subnorm_shard_ymax)

TRAILER = 32


def shard_rows(packed: torch.Tensor, N: int, K: int, r0: int, r1: int) -> torch.Tensor:
    """The I2_S tensor of rows [r0, r1) of an I2_S tensor [N, K]: those rows' bytes followed
    by the original trailer (the whole tensor's scale)."""
    rb = K // 4
    if not (0 <= r0 < r1 <= N) or packed.numel() != i2s_packed_bytes(N, K):
        raise ValueError("bad row range or packed size")
    return torch.cat([packed[r0 * rb:r1 * rb], packed[N * rb:N * rb + TRAILER]]).contiguous()


def shard_cols(packed: torch.Tensor, N: int, K: int, k0: int, k1: int) -> torch.Tensor:
    """The I2_S tensor of in-features [k0, k1) of every row (k0, k1 multiples of 128, so the
    slice is whole 128-weight blocks), followed by the original trailer."""
    if k0 % 128 or k1 % 128 or not (0 <= k0 < k1 <= K) or packed.numel() != i2s_packed_bytes(N, K):
        raise ValueError("column range must be whole 128-weight blocks inside the row")
    rb = K // 4
    body = packed[:N * rb].view(N, rb)[:, k0 // 4:k1 // 4].reshape(-1)
    return torch.cat([body, packed[N * rb:N * rb + TRAILER]]).contiguous()


@dataclasses.dataclass
class FFNShard:
    """One rank's part of an FFN block: intermediate columns [i0, i1)."""
    H: int
    I: int
    i0: int
    i1: int
    p_gate: torch.Tensor
    p_up: torch.Tensor
    p_down: torch.Tensor
    g_sub: torch.Tensor | None

    @property
    def Is(self) -> int:
        return self.i1 - self.i0


def shard_range(I: int, rank: int, world: int) -> tuple[int, int]:
    """Intermediate columns of `rank`: contiguous blocks of whole 128-weight I2_S blocks."""
    if I % (128 * world):
        raise ValueError(f"I = {I} must split into whole 128-wide blocks over {world} ranks")
    w = I // world
    return rank * w, (rank + 1) * w


def make_shard(p_gate, p_up, p_down, g_sub, H: int, I: int, rank: int, world: int) -> FFNShard:
    """Cut this rank's shard out of the whole packed FFN (gate/up [I, H], down [H, I])."""
    i0, i1 = shard_range(I, rank, world)
    return FFNShard(H, I, i0, i1, shard_rows(p_gate, I, H, i0, i1), shard_rows(p_up, I, H, i0, i1),
                    shard_cols(p_down, H, I, i0, i1), None if g_sub is None else g_sub[i0:i1].contiguous())


class ShardRun:
    """The FFN on one shard, in the stages between which the ranks combine their partial
    results (see the module docstring)."""

    def __init__(self, shard: FFNShard, x: torch.Tensor, g_ffn, act: int, eps: float):
        self.sh, self.eps = shard, eps
        q, s, sq = rmsnorm_quant_act(x, g_ffn, eps)  # x is replicated: every rank quantises it
        self.h = bitlinear_gate_up_act(q, s, sq, shard.p_gate, shard.p_up, shard.Is, act)

    def amax(self) -> torch.Tensor:
        return subnorm_shard_amax(self.h)

    def sumsq(self, amax: torch.Tensor):
        if self.sh.g_sub is None:
            return None
        return subnorm_shard_sumsq(self.h, amax, self.sh.I)

    def ymax(self, amax: torch.Tensor, S) -> torch.Tensor:
        self.inv, ym = subnorm_shard_ymax(self.h, self.sh.g_sub, amax, S, self.sh.I, self.eps)
        return ym

    def down_acc(self, ymax: torch.Tensor) -> torch.Tensor:
        self.q_h, self.s_h, self.sum_h = subnorm_shard_quant(self.h, self.sh.g_sub, self.inv, ymax)
        return bitlinear_acc(self.q_h, self.sum_h, self.sh.p_down, self.sh.H)

    def finish(self, acc: torch.Tensor, out_dtype=torch.bfloat16) -> torch.Tensor:
        return dequant_acc(acc, self.s_h, self.sh.p_down, self.sh.Is, out_dtype)


def _dist_max(t: torch.Tensor, group=None) -> torch.Tensor:
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX, group=group)
    return t


def _dist_sum(t: torch.Tensor, group=None) -> torch.Tensor:
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM, group=group)
    return t


def ffn_block_tp(shard: FFNShard, x: torch.Tensor, g_ffn, act: int, eps: float = 1e-6, out_dtype=torch.bfloat16,
                 group=None, reduce_max=None, reduce_sum=None) -> torch.Tensor:
    """The FFN block on this rank's shard; every rank of `group` calls it with the same x
    and gets the same output [T, H] (bit-identical to the single-GPU ffn_block).  Four
    collectives per call, in the same order on every rank: MAX, SUM (int64; skipped when
    ffn_sub_norm is off), MAX, SUM (int32 [T, H])."""
    rmax = reduce_max or (lambda t: _dist_max(t, group))
    rsum = reduce_sum or (lambda t: _dist_sum(t, group))
    run = ShardRun(shard, x, g_ffn, act, eps)
    amax = rmax(run.amax())
    S = run.sumsq(amax)
    if S is not None:
        S = rsum(S)
    ymax = rmax(run.ymax(amax, S))
    acc = rsum(run.down_acc(ymax))
    return run.finish(acc, out_dtype)
