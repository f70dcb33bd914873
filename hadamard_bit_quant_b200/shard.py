"""Token sharding across ranks (one process per GPU).

Every token row of the H-BitLinear forward is independent (its own Hadamard
transform and scale) and the weights are shared, so a global batch splits by
rows with no exchange in the data path. These helpers hold the host-side
logic: the row split, the optional gather of the row-sharded output, and the
max-over-ranks reduction of device timings.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def row_range(M: int, rank: int, world: int):
    """Contiguous, balanced [start, stop) rows of a batch of M tokens for this rank."""
    if world < 1 or not (0 <= rank < world) or M < 0:
        raise ValueError((M, rank, world))
    base, rem = divmod(M, world)
    start = rank * base + min(rank, rem)
    return start, start + base + (1 if rank < rem else 0)


def gather_rows(y_local: torch.Tensor, M: int, group=None) -> torch.Tensor:
    """All-gather row shards (split by ``row_range``) into the full M x N output on every rank."""
    world = dist.get_world_size(group)
    counts = [row_range(M, r, world) for r in range(world)]
    rows = max(b - a for a, b in counts)
    pad = torch.zeros((rows,) + tuple(y_local.shape[1:]), dtype=y_local.dtype, device=y_local.device)
    pad[: y_local.shape[0]] = y_local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[: b - a] for p, (a, b) in zip(parts, counts)], dim=0)


def max_over_ranks(value: float, device=None, group=None) -> float:
    """Max of a per-rank scalar (e.g. a CUDA-event time) over all ranks."""
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
