"""Column-parallel (N-split) decomposed matmul over the ranks of a process group.

The LLM.int8() pages run large models on several GPUs by placing parts of the
model on each ("LLM.int8()", brain.gartu.xyz, section "Exemple pratique":
``device_map="auto"``).  For one layer, the split that needs no exchange
inside the method is by output columns:

* every rank holds the int8 codes, the column scales c_w and the fp16 rows of
  its own contiguous slice of W's columns;
* every rank receives the whole X and finds the outlier set O and the row
  scales c_x itself: both depend on X alone ("LLM.int8() — 大模型激活值里藏着几
  个超大异常通道", 方法1 and 方法2), so all ranks agree on them without talking;
* every rank computes its columns of Y with the single-GPU kernels, and one
  all-gather (NCCL over NVLink on GPUs) assembles the full Y.

Column j of Y depends only on X, W[:, j] and c_w[j], and the int32
accumulators are exact, so the sharded Y equals the unsharded one.

This module holds tensors and calls the C ABI and ``torch.distributed``; all
arithmetic of the method runs in the library's kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (int8mm_forward_bias, int8mm_prepare_weight, int8mm_prepare_weight_static)

ALIGN = 16  # the kernels take N in multiples of 16


def column_ranges(N: int, world: int, align: int = ALIGN) -> list[tuple[int, int]]:
    """Contiguous column slices [n0, n1) of an N-column weight for `world`
    ranks: multiples of `align`, widths differing by at most `align`."""
    if world < 1:
        raise ValueError("world must be >= 1")
    if N % align != 0 or N < align * world:
        raise ValueError(f"N={N} must be a multiple of {align} and at least {align} per rank ({world} ranks)")
    base, extra = divmod(N // align, world)
    ranges, n0 = [], 0
    for r in range(world):
        n1 = n0 + (base + (1 if r < extra else 0)) * align
        ranges.append((n0, n1))
        n0 = n1
    return ranges


def _world_and_rank(group):
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(group), dist.get_rank(group)
    return 1, 0


def gather_columns(Y_local: torch.Tensor, ranges: list[tuple[int, int]], group=None) -> torch.Tensor:
    """All-gather the ranks' column slices of Y ([M, n1 - n0] each, in rank
    order) into the full [M, N] on every rank.  Slices of unequal width are
    padded to the widest for the collective."""
    world, rank = _world_and_rank(group)
    if len(ranges) != world:
        raise ValueError(f"{len(ranges)} column ranges for {world} ranks")
    a, b = ranges[rank]
    if Y_local.dim() != 2 or Y_local.shape[1] != b - a:
        raise ValueError(f"rank {rank} holds columns [{a}, {b}); got Y_local of shape {tuple(Y_local.shape)}")
    if world == 1:
        return Y_local
    M = Y_local.shape[0]
    width = max(n1 - n0 for n0, n1 in ranges)
    send = Y_local.contiguous()
    if b - a != width:
        send = torch.zeros((M, width), dtype=Y_local.dtype, device=Y_local.device)
        send[:, : b - a].copy_(Y_local)
    parts = [torch.empty((M, width), dtype=Y_local.dtype, device=Y_local.device) for _ in range(world)]
    dist.all_gather(parts, send, group=group)
    Y = torch.empty((M, ranges[-1][1]), dtype=Y_local.dtype, device=Y_local.device)
    for r, (n0, n1) in enumerate(ranges):
        Y[:, n0:n1].copy_(parts[r][:, : n1 - n0])
    return Y


class ColumnParallelInt8Matmul:
    """Y = X W with W's columns split over the ranks of `group` (all ranks
    when None; a single process without a process group is one rank).

    Build it on every rank with the full fp16 weight W [K, N] (each rank keeps
    only a copy of its own columns) or with ``from_shard``.  ``static_rows``
    selects the memory-saving weight (int8mm_prepare_weight_static) on every
    rank."""

    def __init__(self, W: torch.Tensor | None, group=None, static_rows=None, max_outliers: int = 256,
                 *, _shard: torch.Tensor | None = None, _N: int | None = None):
        self.group = group
        self.world, self.rank = _world_and_rank(group)
        if _shard is None:
            if W is None or W.dim() != 2:
                raise ValueError("W must be a 2-D fp16 tensor [K, N]")
            N = W.shape[1]
            self.ranges = column_ranges(N, self.world)
            a, b = self.ranges[self.rank]
            shard = W[:, a:b].contiguous()
        else:
            N = _N
            self.ranges = column_ranges(N, self.world)
            a, b = self.ranges[self.rank]
            if _shard.dim() != 2 or _shard.shape[1] != b - a:
                raise ValueError(f"rank {self.rank} holds columns [{a}, {b}); got a shard of shape "
                                 f"{tuple(_shard.shape)}")
            shard = _shard.contiguous()
        self.N = N
        self.K = shard.shape[0]
        self.cols = (a, b)
        if static_rows is None:
            self.shard = shard  # borrowed by the handle: keep it alive
            self.weight = int8mm_prepare_weight(shard)
        else:
            self.shard = None   # the static weight keeps what it needs
            self.weight = int8mm_prepare_weight_static(shard, list(static_rows), max_outliers)

    @classmethod
    def from_shard(cls, shard: torch.Tensor, N: int, group=None, static_rows=None, max_outliers: int = 256):
        """Build from this rank's own columns W[:, n0:n1] of an N-column
        weight (the slice column_ranges(N, world)[rank])."""
        return cls(None, group, static_rows, max_outliers, _shard=shard, _N=N)

    def local_forward(self, X: torch.Tensor, alpha: float = 6.0, bias: torch.Tensor | None = None) -> torch.Tensor:
        """This rank's columns of Y, [M, n1 - n0] (bias: the full [N] bias)."""
        a, b = self.cols
        return int8mm_forward_bias(self.weight, X, alpha, None if bias is None else bias[a:b].contiguous())

    def forward(self, X: torch.Tensor, alpha: float = 6.0, bias: torch.Tensor | None = None) -> torch.Tensor:
        """The full Y [M, N] on every rank (X replicated on all ranks)."""
        return gather_columns(self.local_forward(X, alpha, bias), self.ranges, self.group)

    __call__ = forward
