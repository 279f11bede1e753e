"""Tensor-parallel sharding of the fused merge and the segmented apply.

Megatron-style sharding needs no new kernel: each rank builds its own plan
over its shards and calls the same entry points.

* Column-parallel linears (q, k, v, gate, up): a rank holds a block of output
  rows, W[o0:o1, :] and B_e[o0:o1, :], and the whole A.  Its merge gives
  exactly rows o0:o1 of W' and its apply gives columns o0:o1 of y: nothing
  is exchanged.
* Row-parallel linears (o, down): a rank holds a block of input columns,
  W[:, i0:i1] and A_e[:, i0:i1], and the whole B.  Its merge gives columns
  i0:i1 of W'.  Its apply, on columns i0:i1 of x, gives
      x_s W_s^T + sum_s g_s (x_s A_s^T) B_s^T,
  and because the expand is linear in the shrink, the sum of the ranks'
  partials is the full y: one all-reduce (sum) of y completes it -- the
  all-reduce a row-parallel layer of the backbone performs anyway.  The
  partials stay fp32 (a plan built with PLAN_Y_F32): rounding each to bf16
  before the sum would cost up to half a bf16 ulp per rank, more than the
  output tolerance where the partials cancel; the sum is rounded once, by the
  library's round_bf16 kernel.  A rank therefore builds two plans, one over
  its column-parallel linears and one (PLAN_Y_F32) over its row-parallel ones.

This module only slices tensors and issues that all-reduce; every
arithmetic step stays in the library's kernels.
"""
from __future__ import annotations

from typing import Tuple

COLUMN = "column"
ROW = "row"
_COLUMN_NAMES = ("q", "k", "v", "gate", "up")
_ROW_NAMES = ("o", "down")


def kind_of(name: str) -> str:
    """Sharding of a targeted linear by its role in a Llama block."""
    if name in _COLUMN_NAMES:
        return COLUMN
    if name in _ROW_NAMES:
        return ROW
    raise ValueError(f"no tensor-parallel rule for linear {name!r}")


def block(n: int, rank: int, world: int) -> Tuple[int, int]:
    """[start, stop) of rank's contiguous share of n; shares stay multiples of
    8 elements (16-byte rows, as the library requires)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} of {world}")
    if n % (8 * world):
        raise ValueError(f"{n} does not split into {world} shares of whole 8-element groups")
    step = n // world
    return rank * step, (rank + 1) * step


def shard_weights(kind: str, W, A, B, rank: int, world: int):
    """Rank's (W, A, B) for one linear.  W [d_out, d_in], A [E, r, d_in],
    B [E, d_out, r].  Column shards are views; row shards of W and A are
    contiguous copies (the library reads rows of d_in elements)."""
    if kind == COLUMN:
        o0, o1 = block(W.shape[0], rank, world)
        return W[o0:o1], A, B[:, o0:o1, :]
    if kind == ROW:
        i0, i1 = block(W.shape[1], rank, world)
        return W[:, i0:i1].contiguous(), A[:, :, i0:i1].contiguous(), B
    raise ValueError(kind)


def shard_input(kind: str, x, rank: int, world: int):
    """Rank's activations for one linear: the whole x for a column-parallel
    linear, its block of input columns for a row-parallel one."""
    if kind == COLUMN:
        return x
    if kind == ROW:
        i0, i1 = block(x.shape[1], rank, world)
        return x[:, i0:i1].contiguous()
    raise ValueError(kind)


def plan_flags(kind: str) -> int:
    """Plan flags for a rank's plan over linears of this kind: fp32 outputs
    (PLAN_Y_F32) for row-parallel partials, bf16 for column-parallel ones."""
    if kind == ROW:
        from adapter_merge_b200 import PLAN_Y_F32
        return PLAN_Y_F32
    if kind == COLUMN:
        return 0
    raise ValueError(kind)


def reduce_output(kind: str, y, out=None, group=None):
    """Complete a rank's apply output.  Column-parallel: y (bf16) is already
    final, the rank's block of output columns.  Row-parallel: y is the rank's
    fp32 partial (PLAN_Y_F32); it is all-reduced (sum, in place), and if `out`
    is given (a bf16 device tensor of y's shape) the sum is rounded once into
    it by the library and `out` is returned, else the summed partial.  Every
    rank must call this in the same order."""
    if kind == COLUMN:
        return y
    if kind != ROW:
        raise ValueError(kind)
    import torch.distributed as dist
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(y, op=dist.ReduceOp.SUM, group=group)
    if out is None:
        return y
    from adapter_merge_b200 import round_bf16
    return round_bf16(y, out)
