"""Multi-GPU plumbing of the routing path (one process per GPU, torch.distributed).

Two uses:
  * data parallel (weak scaling): every rank routes its own batch; the only cross-rank step is
    the max over ranks of the measured device time (``max_over_ranks``);
  * expert parallel: every rank routes the same tokens with its own ``expert_map`` (a contiguous
    block of experts, ``ep_expert_map``); its combine is the partial sum over its local slots, and
    the one exchange of the layer is the sum of those partials over the ranks
    (``ep_reduce_partials``: fp32 sum of the bf16 partials, rounded once to bf16).

The exchange follows the expert-parallel decode of the "b70-optimization-lab: 2026-07-16 MTP1
M=2 compact scheduler closure note" (scheduler paragraph: each rank derives its local expert row
counts from topk_ids plus expert_map; the collective is left out there and done here).
"""
from __future__ import annotations

import os
from typing import Optional, Tuple

import torch
import torch.distributed as dist


def rank_env() -> Tuple[int, int, int]:
    """(world size, rank, local rank) from the launcher's environment (1, 0, 0 without one)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s batch in a data-parallel run: an independent batch per rank."""
    return seed + rank


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of `value` over all ranks (the value itself without a process group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def ep_expert_range(E: int, world: int, rank: int) -> Tuple[int, int]:
    """Global experts [lo, hi) owned by `rank` when E experts are split into `world` contiguous
    blocks (the first E % world ranks own one more)."""
    if world < 1 or not 0 <= rank < world or E < world:
        raise ValueError(f"cannot split {E} experts over {world} ranks (rank {rank})")
    base, extra = divmod(E, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def ep_expert_map(E: int, world: int, rank: int) -> Tuple[torch.Tensor, int]:
    """(int32 [E] global -> local map of `rank`, -1 for the other ranks' experts; E_local)."""
    lo, hi = ep_expert_range(E, world, rank)
    m = torch.full((E,), -1, dtype=torch.int32)
    m[lo:hi] = torch.arange(hi - lo, dtype=torch.int32)
    return m, hi - lo


def ep_reduce_partials(partial: torch.Tensor, group: Optional[dist.ProcessGroup] = None) -> torch.Tensor:
    """Sum the ranks' bf16 partial combines [T, H]: widened to fp32, summed over the ranks, rounded
    once to bf16 (round-to-nearest-even).  Returns a new tensor; with one rank, the partial."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return partial.clone()
    acc = partial.float()
    dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=group)
    return acc.to(torch.bfloat16)
