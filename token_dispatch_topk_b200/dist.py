"""Multi-GPU plumbing of the routing path (one process per GPU, torch.distributed).

Two uses:
  * data parallel (weak scaling): every rank routes its own batch; the only cross-rank step is
    the max over ranks of the measured device time (``max_over_ranks``);
  * expert parallel: every rank routes the same tokens with its own ``expert_map`` (a contiguous
    block of experts, ``ep_expert_map``); its combine is the partial sum over its local slots, and
    the one exchange of the layer is the sum of those partials over the ranks: fp32 sum of the bf16
    partials in ascending rank order, rounded once to bf16.  Two forms:
      - ``EpExchange`` (the library's form, a reduce-scatter): each rank's moe_combine writes each
        owner's token range (``ep_token_range``) of its partial straight into its slot of that
        owner's receive buffer, in the owner's memory, shared between the processes through CUDA IPC
        and mapped in each rank's own device context (on several GPUs the combine's own stores cross
        NVLink; plain 16-byte stores, no TMA, no multicast); each rank then synchronises its stream and joins a process-group barrier, so
        that every store into every owner's buffer has completed before any owner reads; then each
        owner runs moe_reduce_partials over its slots in rank order.  Two receive buffers alternate
        between steps, so one barrier per step also keeps a step's stores away from the buffer the
        owner is still reducing from the step before;
      - ``ep_reduce_partials``: an all-gather of the whole partials through the process group, then
        the same rank-ordered reduce on every rank (bit-identical to the reduce-scatter's rows; the
        collective baseline).
    ``ep_combine_to_owners`` and ``ep_reduce_received`` are the two halves of the reduce-scatter for
    callers that manage their own buffers; a caller must order every rank's combine before the
    owners' reduces (synchronise the combine's stream, or wait on its event, before a barrier).

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


def _share(t: torch.Tensor):
    """A picklable CUDA IPC handle of a device tensor (torch's own sharing of CUDA storage)."""
    from torch.multiprocessing.reductions import reduce_tensor
    return reduce_tensor(t)


def _check_peer_access(device, group: Optional[dist.ProcessGroup] = None) -> None:
    """Every rank's device must reach every other rank's device directly (NVLink or PCIe peer access)
    before buffers are shared: the kernels read and write the peers' memory with plain loads and stores.
    Raises on this rank when one cannot; gathers the ranks' device indices through the process group."""
    me = torch.device(device).index
    me = torch.cuda.current_device() if me is None else me
    devs = [None] * dist.get_world_size(group)
    dist.all_gather_object(devs, me, group=group)
    for d in devs:
        if d != me and not torch.cuda.can_device_access_peer(me, d):
            raise RuntimeError(f"device {me} cannot access device {d} directly: no shared receive buffers")


def _open_shared(handle, device) -> torch.Tensor:
    """Map another process's tensor (a handle from ``_share``) into this process, opened in the context
    of this rank's own device: the mapping is then this device's, with peer access enabled as needed,
    so this device's kernels may read and write it (over NVLink when it lives on another GPU).  The
    tensor reports this device; its memory is the other process's.  The owner synchronised its device
    before sharing and the handles travel through the process group afterwards, so no IPC event is
    opened to order the first use."""
    from torch.multiprocessing.reductions import rebuild_cuda_tensor
    fn, args = handle
    if fn is not rebuild_cuda_tensor or len(args) != 15:
        raise RuntimeError("unexpected CUDA IPC handle layout")
    args = list(args)
    args[6] = torch.device(device).index if torch.device(device).index is not None else torch.cuda.current_device()
    args[14] = False  # event_sync_required
    return fn(*args)


def ep_reduce_partials(partial: torch.Tensor, group: Optional[dist.ProcessGroup] = None,
                       reduce=None) -> torch.Tensor:
    """Sum the ranks' bf16 partial combines [T, H] (the collective baseline of the exchange): an
    all-gather of every rank's partial, then the fp32 sum in ascending rank order from +0, rounded
    once to bf16, on every rank.  ``reduce`` maps the list of partials (rank order) to the sum;
    default: moe_reduce_partials on the partials' device.  Returns a new tensor; with one rank, a
    copy of the partial."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return partial.clone()
    parts = [torch.empty_like(partial) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, partial.contiguous(), group=group)
    if reduce is None:
        from .binding import moe_reduce_partials
        return moe_reduce_partials(parts)
    return reduce(parts)


class EpExchange:
    """The expert-parallel exchange as a reduce-scatter through the owners' memory (see the module
    docstring).  One object per rank, created by every rank of ``group`` together (it exchanges
    CUDA IPC handles of the receive buffers through the process group).

    ``combine_reduce(expert_out, topk_weights, inv_perm)`` runs one step: this rank's partial combine
    into every owner's receive buffer, the barrier, and this owner's reduce; it returns this owner's
    rows of the layer output ([hi - lo, H] bf16 for ``ep_token_range(T, world, rank)``), in a buffer the
    next step overwrites.  Without a process group it is a single rank's exchange (its own buffer)."""

    def __init__(self, T: int, H: int, device, group: Optional[dist.ProcessGroup] = None, buffers: int = 2):
        self.group = group
        grouped = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if grouped else 1  # one rank: its own buffer, no barrier
        self.rank = dist.get_rank(group) if grouped else 0
        self.T, self.H = T, H
        self.ranges = [ep_token_range(T, self.world, o) for o in range(self.world)]
        lo, hi = self.ranges[self.rank]
        rows = max(1, hi - lo)  # every owner shares a buffer, even one without tokens
        self.recv = [torch.zeros((self.world, rows, H), dtype=torch.bfloat16, device=device) for _ in range(buffers)]
        self.out = torch.empty((hi - lo, H), dtype=torch.bfloat16, device=device)
        torch.cuda.synchronize(device)
        if self.world > 1:
            _check_peer_access(device, group)
            mine = [_share(b) for b in self.recv]
            handles = [None] * self.world
            dist.all_gather_object(handles, mine, group=group)
            # remote[b][o]: owner o's receive buffer b, as mapped in this process
            self.remote = [[self.recv[b] if o == self.rank else _open_shared(handles[o][b], device)
                            for o in range(self.world)] for b in range(buffers)]
            dist.barrier(group=group)
        else:
            self.remote = [[b] for b in self.recv]
        self.step_index = 0

    def destinations(self, b: int):
        """This rank's slot in every owner's receive buffer b (owner order)."""
        return [self.remote[b][o][self.rank, :hi - lo] for o, (lo, hi) in enumerate(self.ranges)]

    def combine_reduce(self, expert_out: torch.Tensor, topk_weights: torch.Tensor, inv_perm: torch.Tensor,
                       device_status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        from .binding import moe_reduce_partials
        b = self.step_index % len(self.recv)
        self.step_index += 1
        s = torch.cuda.current_stream() if stream is None else stream
        ep_combine_to_owners(expert_out, topk_weights, inv_perm, self.destinations(b), device_status=device_status,
                             stream=s)
        if self.world > 1:
            s.synchronize()                 # this rank's stores into every owner's buffer have completed
            dist.barrier(group=self.group)  # ... and every other rank's into this owner's
        lo, hi = self.ranges[self.rank]
        if hi > lo:
            moe_reduce_partials([self.recv[b][r, :hi - lo] for r in range(self.world)], out=self.out, stream=s)
        return self.out


class EpAllToAll:
    """The expert-parallel layer with the tokens sharded over the ranks (the all-to-all form).

    Rank r holds its own T_r tokens (``T_per_rank[r]``) and owns a contiguous block of experts.  One
    ``step`` on every rank:
      1. gating of this rank's tokens (moe_topk_softmax) into buffers the other ranks can read;
      2. a barrier; each owner copies every rank's routes into one list (one peer copy per rank), aligns
         them with its expert_map (moe_align_permute: the expert-grouped layout of every rank's slots
         on its experts, rank by rank in slot order) and pulls the hidden rows it needs from each rank
         (moe_gather with that rank's hidden rows as the source: bulk loads from the rank's memory);
      3. the owner's experts run on the expert-grouped rows (``expert_out`` stands in for them here);
      4. for every rank, the owner's moe_combine of that rank's slots on its experts is written straight
         into the rank's receive buffer (stores into the rank's memory);
      5. a barrier; each rank reduces its partials in ascending owner order (moe_reduce_partials): the
         same sum as the replicated-token exchange (fp32 in rank order, rounded once to bf16).
    The buffers other ranks read or write (routes, weights, hidden rows, receive buffers) are shared
    through CUDA IPC.  The caller writes this step's hidden rows into ``hidden`` before ``step``.
    Returns this rank's layer output [T_r, H] (overwritten by the next step).  Without a process
    group it is a single rank's layer (its own buffers, no barrier)."""

    def __init__(self, T_per_rank, E: int, k: int, H: int, block_size: int, renormalize: bool, device,
                 group: Optional[dist.ProcessGroup] = None, logits_dtype=torch.bfloat16):
        from . import binding as B
        self.group = group
        grouped = dist.is_available() and dist.is_initialized()
        self.world = dist.get_world_size(group) if grouped else 1  # one rank: its own buffers, no barrier
        self.rank = dist.get_rank(group) if grouped else 0
        assert len(T_per_rank) == self.world
        self.T = list(int(t) for t in T_per_rank)
        self.off = [sum(self.T[:r]) for r in range(self.world)]
        self.T_total = sum(self.T)
        self.E, self.k, self.H, self.block_size, self.renormalize = E, k, H, block_size, renormalize
        emap, self.E_local = ep_expert_map(E, self.world, self.rank)
        self.expert_map = emap.to(device)
        Tr = self.T[self.rank]
        # shared with the other ranks
        self.topk_ids = torch.zeros((max(1, Tr), k), dtype=torch.int32, device=device)
        self.topk_weights = torch.zeros((max(1, Tr), k), dtype=torch.float32, device=device)
        self.hidden = torch.zeros((max(1, Tr), H), dtype=torch.bfloat16, device=device)
        self.recv = torch.zeros((self.world, max(1, Tr), H), dtype=torch.bfloat16, device=device)
        # this owner's own
        self.ids_all = torch.zeros((max(1, self.T_total), k), dtype=torch.int32, device=device)
        self.align = B.alloc_align_outputs(self.T_total, k, self.E_local, block_size, device)
        self.capacity = self.align.capacity
        self.workspace = B.alloc_workspace(self.T_total, k, self.E_local, device)
        self.permuted = torch.empty((self.capacity, H), dtype=torch.bfloat16, device=device)
        self.out = torch.empty((Tr, H), dtype=torch.bfloat16, device=device)
        torch.cuda.synchronize(device)
        own = (self.topk_ids, self.topk_weights, self.hidden, self.recv)
        if self.world > 1:
            _check_peer_access(device, group)
            mine = [_share(t) for t in own]
            handles = [None] * self.world
            dist.all_gather_object(handles, mine, group=group)
            peers = [own if o == self.rank else tuple(_open_shared(h, device) for h in handles[o])
                     for o in range(self.world)]
            dist.barrier(group=group)
        else:
            peers = [own]
        self.peer_ids, self.peer_w, self.peer_hidden, self.peer_recv = (list(x) for x in zip(*peers))

    def slots(self, r: int) -> slice:
        """Rank r's slots in this owner's list of every rank's routes."""
        return slice(self.off[r] * self.k, (self.off[r] + self.T[r]) * self.k)

    def step(self, logits: torch.Tensor, expert_out: torch.Tensor, stream=None) -> torch.Tensor:
        from . import binding as B
        s = torch.cuda.current_stream() if stream is None else stream
        Tr, k = self.T[self.rank], self.k
        with torch.cuda.stream(s):
            if Tr:
                B.moe_topk_softmax(logits, k, self.renormalize, self.topk_weights[:Tr], self.topk_ids[:Tr], s)
            if self.world > 1:
                s.synchronize()
                dist.barrier(group=self.group)  # every rank's routes and hidden rows are ready
            for r in range(self.world):
                if self.T[r]:
                    self.ids_all[self.off[r]:self.off[r] + self.T[r]].copy_(self.peer_ids[r][:self.T[r]],
                                                                            non_blocking=True)
            B.moe_align_permute(self.ids_all[:self.T_total], self.E, self.block_size, self.expert_map, self.E_local,
                                self.align, self.workspace, s)
            inv = self.align.inv_perm
            for r in range(self.world):
                if self.T[r]:
                    B.moe_gather(self.peer_hidden[r][:self.T[r]], k, inv[self.slots(r)], self.capacity,
                                 permuted=self.permuted, device_status=self.workspace, stream=s)
            # (the owner's experts run here on self.permuted; expert_out stands in for their output)
            for r in range(self.world):
                if self.T[r]:
                    B.moe_combine(expert_out, self.peer_w[r][:self.T[r]], inv[self.slots(r)],
                                  self.peer_recv[r][self.rank, :self.T[r]], device_status=self.workspace, stream=s)
            if self.world > 1:
                s.synchronize()
                dist.barrier(group=self.group)  # every owner's partial for every rank has landed
            if Tr:
                B.moe_reduce_partials([self.recv[o, :Tr] for o in range(self.world)], out=self.out, stream=s)
        return self.out
