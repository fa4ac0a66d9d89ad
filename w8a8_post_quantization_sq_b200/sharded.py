"""Sharded calibration across data-parallel ranks.

Quantisation and the GEMMs are independent per token row, so data-parallel
replicas need no collective. Calibration is the exception: x_j is the maximum
of |X_j| over all calibration tokens ("大语言模型量化技术（四）：SmoothQuant",
section 缩放因子). Here each rank takes the running maxima over its own shard
of the calibration batches (batch i goes to rank i mod world) with one of the
library's calibration calls, then the ranks exchange them once: the
element-wise maximum over the ranks. A maximum is exact and order-free, so
every rank ends with the bits one device would get from all the batches.
"""
from __future__ import annotations

from typing import Callable, Sequence

import torch
import torch.distributed as dist


def _rank_world(group=None):
    if dist.is_available() and dist.is_initialized():
        return dist.get_rank(group), dist.get_world_size(group)
    return 0, 1


def shard(n_batches: int, rank: int, world: int) -> range:
    """The calibration batches of `rank`: i = rank, rank + world, ..."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    return range(rank, n_batches, world)


def allreduce_max_(maxima: torch.Tensor, group=None) -> torch.Tensor:
    """In place: maxima <- element-wise max over the ranks of `group` (NCCL for
    CUDA tensors, gloo for CPU ones). Returns the tensor."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(maxima, op=dist.ReduceOp.MAX, group=group)
    return maxima


def calibrate_sharded(batches: Sequence, maxima: torch.Tensor, update: Callable, group=None) -> torch.Tensor:
    """Running maxima over this rank's shard of `batches`, then their maximum
    over the ranks, in place in `maxima` (which starts at zero, or at earlier
    maxima to extend). `update(batch, maxima)` folds one batch into the
    running maxima: sq_calib_absmax for the linear inputs themselves, or the
    calibration mode of sq_norm_smooth_quant / sq_act_quant wrapped to that
    form. Every rank must call this with the same number of batches."""
    rank, world = _rank_world(group)
    for i in shard(len(batches), rank, world):
        update(batches[i], maxima)
    return allreduce_max_(maxima, group)
