"""Multi-GPU plumbing of the routing path (one process per GPU, torch.distributed).

Two uses:
  * data parallel (weak scaling): every rank routes its own batch; the only cross-rank step is
    the max over ranks of the measured device time (``max_over_ranks``);
  * expert parallel: every rank routes the same tokens with its own ``expert_map`` (a contiguous
    block of experts, ``ep_expert_map``); its combine is the partial sum over its local slots, and
    the one exchange of the layer is the sum of those partials over the ranks: fp32 sum of the bf16
    partials, rounded once to bf16.  Two forms:
      - ``ep_reduce_partials``: an NCCL all-reduce of the widened partials;
      - reduce-scatter through the library: ``ep_combine_to_owners`` (each rank's combine writes each
        owner's token range into the owner's receive buffer, ``ep_token_range``), then, after a
        barrier, ``ep_reduce_received`` on every owner (moe_reduce_partials, rank order).  The
        receive buffers of a multi-GPU run are peer memory (e.g. symmetric memory); the tests run
        the ranks on one GPU with local buffers in their place.

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


def ep_token_range(T: int, world: int, owner: int) -> Tuple[int, int]:
    """Tokens [lo, hi) whose layer output rank `owner` assembles in the reduce-scatter form of the
    exchange (contiguous blocks, the first T % world owners one token more; empty when T < world)."""
    if world < 1 or not 0 <= owner < world or T < 0:
        raise ValueError(f"cannot split {T} tokens over {world} ranks (owner {owner})")
    base, extra = divmod(T, world)
    lo = owner * base + min(owner, extra)
    return lo, lo + base + (1 if owner < extra else 0)


def ep_combine_to_owners(expert_out: torch.Tensor, topk_weights: torch.Tensor, inv_perm: torch.Tensor,
                         destinations, device_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """This rank's part of the reduce-scatter: its partial combine, each owner's token range written
    straight into `destinations[owner]` ([hi - lo, H] bf16, this rank's slot in the owner's receive
    buffer; on a multi-GPU run a tensor in the owner's memory, reached over NVLink by the combine's
    own stores).  topk_weights [T, k] and inv_perm [T*k] are this rank's, from its expert_map."""
    from .binding import moe_combine
    T, k = topk_weights.shape
    world = len(destinations)
    for owner in range(world):
        lo, hi = ep_token_range(T, world, owner)
        if hi > lo:
            moe_combine(expert_out, topk_weights[lo:hi], inv_perm[lo * k:hi * k], out=destinations[owner],
                        device_status=device_status, stream=stream)


def ep_reduce_received(received, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The owner's part of the reduce-scatter, once every rank has written its slot: the fp32 sum in
    rank order of the partials received from the ranks (list in rank order), rounded once to bf16."""
    from .binding import moe_reduce_partials
    return moe_reduce_partials(received, out=out, stream=stream)


def ep_reduce_partials(partial: torch.Tensor, group: Optional[dist.ProcessGroup] = None) -> torch.Tensor:
    """Sum the ranks' bf16 partial combines [T, H]: widened to fp32, summed over the ranks, rounded
    once to bf16 (round-to-nearest-even).  Returns a new tensor; with one rank, the partial."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return partial.clone()
    acc = partial.float()
    dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=group)
    return acc.to(torch.bfloat16)
