"""Data-parallel plumbing around the activation path.

The path is elementwise, so it shards without any exchange: each rank applies
the kernels to its own slice of the batch (or its own batch) and the outputs
y and dx never leave the rank.  The only cross-rank step is the combine of
the parameter gradients of the learnable variants (Swish's d alpha, the fused
affine's d gamma / d beta), which in data-parallel training are ordinary
parameter gradients.  To keep them bitwise reproducible for a given world
size, every rank all-gathers the per-rank partials and adds them in rank
order in fp64, so all ranks hold identical bits.  torch.distributed carries
the data (NCCL over NVLink on GPUs, gloo on CPUs); the partials are a handful
of floats, so the collective is latency-bound.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

# Shard boundaries are multiples of this many elements, so that every shard of
# a 16-byte-aligned tensor starts 16-byte aligned (the kernels' vector path).
SHARD_ALIGN = 256


def shard_range(n: int, rank: int, world: int, align: int = SHARD_ALIGN) -> tuple[int, int]:
    """[start, end) of rank's contiguous slice of n elements: slices differ in
    size by at most `align` elements, every start is a multiple of `align`, and
    together they cover [0, n) exactly once."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    if n < 0:
        raise ValueError("n must be non-negative")
    units = (n + align - 1) // align
    lo = units * rank // world
    hi = units * (rank + 1) // world
    return min(lo * align, n), min(hi * align, n)


def combine_param_grads(local: torch.Tensor, group=None) -> torch.Tensor:
    """Sum of every rank's `local` (same shape on all ranks), added in rank
    order in fp64 and returned in local's dtype; identical bits on every rank."""
    world = dist.get_world_size(group)
    flat = local.detach().reshape(-1).to(torch.float64).contiguous()
    gathered = [torch.empty_like(flat) for _ in range(world)]
    dist.all_gather(gathered, flat, group=group)
    acc = gathered[0].clone()
    for r in range(1, world):
        acc += gathered[r]
    return acc.to(local.dtype).reshape(local.shape)


def max_over_ranks(value: float, device: torch.device | str = "cpu", group=None) -> float:
    """Largest `value` over the ranks (for timing: the slowest rank sets the time)."""
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
