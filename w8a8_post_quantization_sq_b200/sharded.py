"""The one exchange of sharded calibration.

Quantisation and the GEMMs are independent per token row, so data-parallel
replicas need no collective. Calibration is the exception: when each rank
collects the running maxima (sq_calib_absmax, sq_weight_absmax, or the
calibration mode of sq_norm_smooth_quant / sq_act_quant) over its own shard of
the calibration tokens, the per-channel maxima of the whole set are the
element-wise maximum over the ranks ("大语言模型量化技术（四）：SmoothQuant",
section 缩放因子: x_j is the max over all calibration tokens). Max is exact and
order-free, so every rank ends with the same bits a single device would get
from all the tokens.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def allreduce_max_(maxima: torch.Tensor, group=None) -> torch.Tensor:
    """In place: maxima <- element-wise max over the ranks of `group` (NCCL for
    CUDA tensors, gloo for CPU ones). Returns the tensor."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(maxima, op=dist.ReduceOp.MAX, group=group)
    return maxima
