"""Host-side helpers for running the attention forward on several GPUs, one
process per GPU (torch.distributed; NCCL on GPUs, gloo in CPU tests).

Attention rows of different (batch, head) pairs are independent, so the work
splits across ranks with no exchange on the data path: each rank runs its own
share of the batch (or of the kv-head groups) and writes a disjoint slice of
the output.  The only collectives are control ones: a barrier and the max of
the ranks' timings, plus an optional gather when a caller wants the whole
output on every rank.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_range(n: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous share [start, end) of n items for `rank` of `world`; the
    first n % world ranks take one extra item."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("rank must be in [0, world)")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def shard_heads(kv_heads: int, group: int, rank: int, world: int) -> tuple[int, int, int, int]:
    """Split whole GQA groups: returns (q_head_start, q_head_end, kv_head_start,
    kv_head_end) for this rank, so every query head keeps its kv head."""
    k0, k1 = shard_range(kv_heads, rank, world)
    return k0 * group, k1 * group, k0, k1


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar (e.g. the timed milliseconds) over all ranks."""
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gather_along(local: torch.Tensor, dim: int = 0) -> torch.Tensor:
    """All ranks' shards concatenated along `dim` (shards may differ in size
    along `dim`, as shard_range gives them)."""
    if not (dist.is_available() and dist.is_initialized()):
        return local
    world = dist.get_world_size()
    sizes = torch.tensor([local.shape[dim]], dtype=torch.int64, device=local.device)
    all_sizes = [torch.zeros_like(sizes) for _ in range(world)]
    dist.all_gather(all_sizes, sizes)
    n_max = int(max(s.item() for s in all_sizes))
    pad = list(local.shape)
    pad[dim] = n_max
    buf = torch.zeros(pad, dtype=local.dtype, device=local.device)
    buf.narrow(dim, 0, local.shape[dim]).copy_(local)
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf)
    return torch.cat([p.narrow(dim, 0, int(s.item())) for p, s in zip(parts, all_sizes)], dim=dim)
