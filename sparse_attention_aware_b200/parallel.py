"""Multi-GPU plumbing for the sparse-attention hot path.

The path partitions into independent problems -- sequences of a decode batch,
query heads (or kv-head groups) of a prefill -- with no exchange step, so N
GPUs run one process each on a contiguous share of the units and no
collective sits on the data path.  torch.distributed (NCCL on GPUs, gloo on
CPU) is used only to agree on timings and to gather results for checking.
"""
from __future__ import annotations

from typing import List, Tuple

import torch
import torch.distributed as dist


def shard_range(n: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous share [lo, hi) of n units for `rank` of `world` (sizes differ
    by at most one; earlier ranks take the extra units)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(n, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def kv_group_shard(num_q_heads: int, num_kv_heads: int, world: int, rank: int) -> Tuple[int, int]:
    """Query-head range of this rank's kv-head groups (prefill sharding keeps a
    GQA group, and so its K/V, on one GPU)."""
    g0, g1 = shard_range(num_kv_heads, world, rank)
    group = num_q_heads // num_kv_heads
    return g0 * group, g1 * group


def max_over_ranks(values: List[float], device=None) -> List[float]:
    """Element-wise max of per-rank values (device times), identical on every
    rank.  Without an initialised process group it returns the input."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def aggregate_throughput(units_per_rank: float, seconds_per_rank: List[float]) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return units_per_rank * len(seconds_per_rank) / max(seconds_per_rank)


def gather_concat(t: torch.Tensor, dim: int = 0) -> torch.Tensor:
    """Concatenate every rank's tensor along `dim` (shapes may differ along dim)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return t
    world = dist.get_world_size()
    n = torch.tensor([t.shape[dim]], dtype=torch.int64, device=t.device)
    sizes = [torch.zeros_like(n) for _ in range(world)]
    dist.all_gather(sizes, n)
    sizes = [int(s.item()) for s in sizes]
    mx = max(sizes)
    pad_shape = list(t.shape)
    pad_shape[dim] = mx - t.shape[dim]
    padded = torch.cat([t, t.new_zeros(pad_shape)], dim=dim) if pad_shape[dim] else t
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded.contiguous())
    return torch.cat([p.narrow(dim, 0, s) for p, s in zip(parts, sizes)], dim=dim)
