"""Data-parallel use of BRA across ranks (one process per GPU).

Images never interact in BRA: routing is an R x R step inside one image and attention
reads only that image's keys. So a batch shards along its image axis with no data-path
collective; each rank runs bra_forward on its own contiguous slice. The only cross-rank
steps here are outside the path: timing (max over ranks) and, when one rank must hold
every output, an all-gather.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_range(B: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous slice [start, stop) of the B images that `rank` of `world` owns; sizes
    differ by at most one, lower ranks take the extra images."""
    if world <= 0 or not 0 <= rank < world or B < 0:
        raise ValueError(f"bad shard request B={B} rank={rank} world={world}")
    base, extra = divmod(B, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device: torch.device | None = None) -> float:
    """The maximum of `value` over all ranks (a timing reduction)."""
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def forward_local(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, n_win: int, topk: int, heads: int,
                  forward_fn=None):
    """Runs the forward pass on this rank's slice of a global batch [B, H, W, C] (which
    may live anywhere; only the slice is used). Returns (start, stop, out, idx)."""
    rank = dist.get_rank() if dist.is_initialized() else 0
    world = dist.get_world_size() if dist.is_initialized() else 1
    start, stop = shard_range(q.shape[0], rank, world)
    if forward_fn is None:
        from .api import forward as forward_fn
    out, idx = forward_fn(q[start:stop].contiguous(), k[start:stop].contiguous(), v[start:stop].contiguous(),
                          n_win, topk, heads)
    return start, stop, out, idx


def gather_images(local: torch.Tensor, B: int) -> torch.Tensor:
    """All-gather of per-rank image slices (as produced by shard_range) into the full batch."""
    world = dist.get_world_size()
    sizes = [shard_range(B, r, world)[1] - shard_range(B, r, world)[0] for r in range(world)]
    width = max(sizes)
    pad = torch.zeros((width, *local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[:local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad)
    return torch.cat([p[:n] for p, n in zip(parts, sizes)], dim=0)
