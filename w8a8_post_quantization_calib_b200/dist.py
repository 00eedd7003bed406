"""Calibration and the linear across ranks (one process per GPU).

Data-parallel calibration: the calibration token batches are sharded over
the ranks; each rank runs sq_calib_absmax on its own shard, and one
all-reduce(MAX) of the K-float statistic makes the per-channel maxima --
hence the smoothing factors, the static activation scale and the weight
codes -- identical on every rank.  This is the quantisation-parameter sync
across cards of pwwt.cn "SmoothQuant技术解析" section 4.3, done on the
statistic (16 KB for K = 4096) instead of on s.  Max is exact and
order-free, so the result equals a single-process calibration over all
shards, bit for bit.

Column-parallel linear (tensor parallelism over the output channels): rank r
holds the weight rows column_shard(N, r, world) and produces those columns
of Y.  The weight column statistic max|W_j| runs over all N rows, so each
rank takes it on its own rows and the same all-reduce(MAX) completes it;
after that s is identical everywhere, the per-row weight scales and codes
of a shard are those of the full matrix, and each output column depends on
its own weight row only: the shards' columns, gathered, equal the
single-process output bit for bit.  No exchange is needed on the forward
path unless the caller wants the full Y on every rank.
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


def column_shard(n_cols: int, rank: int, world: int, multiple: int = 16) -> tuple[int, int]:
    """[start, stop) of rank's output channels for a column-parallel linear:
    whole groups of `multiple` channels (the GEMM takes N a multiple of 16),
    shared as evenly as shard_range shares items."""
    if n_cols % multiple:
        raise ValueError("n_cols must be a multiple of `multiple`")
    a, b = shard_range(n_cols // multiple, rank, world)
    return a * multiple, b * multiple


def allgather_columns(y_local: torch.Tensor, n_cols: int, group=None) -> torch.Tensor:
    """Concatenate every rank's column shard [M, n_r] of a column-parallel
    output into the full [M, n_cols] (ranks in order; shards per column_shard)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return y_local
    world = dist.get_world_size(group)
    spans = [column_shard(n_cols, r, world) for r in range(world)]
    width = max(b - a for a, b in spans)             # equal-size buffers for the collective
    m = y_local.shape[0]
    send = torch.zeros((m, width), dtype=y_local.dtype, device=y_local.device)
    send[:, :y_local.shape[1]] = y_local
    parts = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(parts, send, group=group)
    return torch.cat([p[:, :b - a] for p, (a, b) in zip(parts, spans)], dim=1)

