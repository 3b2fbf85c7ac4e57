"""Data-parallel use of the forward across GPUs: one process per GPU.

Output pixels depend only on their own image (its x and its offset_mask), so a
batch splits across ranks along N with no exchange at all; each rank runs the
forward on its contiguous share of images. Only when every rank needs the
whole result do the ranks exchange it, with one all-gather of the output
shares (NCCL over NVLink on GPUs). Spatial splitting of one image is not
offered: its halo depends on the offsets, which are unbounded.
"""
from __future__ import annotations

from typing import Callable

import torch
import torch.distributed as dist


def batch_shard(N: int, world_size: int, rank: int) -> tuple[int, int]:
    """Contiguous [start, stop) of images for `rank`; shares differ by at most one image."""
    if world_size <= 0 or not 0 <= rank < world_size or N < 0:
        raise ValueError("invalid N / world_size / rank")
    base, extra = divmod(N, world_size)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, group=None, device=None) -> float:
    """The largest `value` over all ranks (a step time is the slowest rank's)."""
    if not dist.is_available() or not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def forward_sharded(x: torch.Tensor, offset_mask: torch.Tensor, G: int, K: int, stride: int = 1, pad: int = 0,
                    dilation: int = 1, offset_scale: float = 1.0, gather: bool = True, group=None,
                    compute: Callable | None = None) -> torch.Tensor:
    """Runs this rank's share of the batch and optionally all-gathers the result.

    x [N,H,W,C] and offset_mask [N,Hout,Wout,G,3K^2] hold the full batch (on
    this rank's device). Returns the full output [N,Hout,Wout,C] when `gather`,
    else this rank's share. `compute` defaults to the CUDA forward.
    """
    if compute is None:
        from .binding import forward as compute
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    N = x.shape[0]
    start, stop = batch_shard(N, world, rank)
    part = compute(x[start:stop].contiguous(), offset_mask[start:stop].contiguous(), G=G, K=K, stride=stride,
                   pad=pad, dilation=dilation, offset_scale=offset_scale)
    if not gather or world == 1:
        return part
    # equal-size pieces for the collective: pad every share to the largest one
    most = batch_shard(N, world, 0)[1]
    padded = torch.zeros((most,) + tuple(part.shape[1:]), dtype=part.dtype, device=part.device)
    padded[:part.shape[0]] = part
    pieces = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(pieces, padded, group=group)
    return torch.cat([pieces[r][:batch_shard(N, world, r)[1] - batch_shard(N, world, r)[0]] for r in range(world)])
