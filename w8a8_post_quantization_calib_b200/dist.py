"""Data-parallel calibration across ranks (one process per GPU).

The calibration token batches are sharded over the ranks; each rank runs
sq_calib_absmax on its own shard, and one all-reduce(MAX) of the K-float
statistic makes the per-channel maxima -- hence the smoothing factors, the
static activation scale and the weight codes -- identical on every rank.
This is the quantisation-parameter sync across cards of pwwt.cn
"SmoothQuant技术解析" section 4.3, done on the statistic (16 KB for K = 4096)
instead of on s.  Max is exact and order-free, so the result equals a
single-process calibration over all shards, bit for bit.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_range(n_items: int, rank: int, world: int) -> tuple[int, int]:
    """[start, stop) of rank's contiguous share of n_items (sizes differ by at most 1)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(n_items, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_absmax_(absmax: torch.Tensor, group=None) -> torch.Tensor:
    """In-place all-reduce(MAX) of a per-channel statistic over the process group."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(absmax, op=dist.ReduceOp.MAX, group=group)
    return absmax
