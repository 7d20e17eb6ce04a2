"""MoeRouter: the routing path for fixed sizes with every buffer preallocated on the device.

One ``step`` runs the routing path on one stream: moe_route_dispatch (gating + align +
permute-gather; one kernel for decode-sized batches, three above) -> (caller's experts) ->
moe_combine.  ``step_staged`` runs the same path through the four stage entry points
moe_topk_softmax -> moe_align_permute -> moe_gather -> moe_combine.
No allocation, host synchronisation or Python-side arithmetic happens inside a step, so
it can be captured in a CUDA graph.  ``step_from_host`` is the end-to-end form: it copies
the step's inputs from (pinned) host memory, runs the step and copies the result back.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import binding as B


class MoeRouter:
    def __init__(self, T: int, E: int, k: int, H: int, block_size: int, renormalize: bool,
                 E_local: Optional[int] = None, expert_map: Optional[torch.Tensor] = None,
                 logits_dtype: torch.dtype = torch.bfloat16, device="cuda", scoring: str = "softmax"):
        B.load_library()
        self.scoring = scoring
        self.T, self.E, self.k, self.H, self.block_size = T, E, k, H, block_size
        self.renormalize = renormalize
        self.E_local = E if E_local is None else E_local
        self.device = torch.device(device)
        self.expert_map = None if expert_map is None else expert_map.to(self.device, torch.int32).contiguous()
        self.logits_dtype = logits_dtype
        self.topk_weights = torch.empty((T, k), dtype=torch.float32, device=self.device)
        self.topk_ids = torch.empty((T, k), dtype=torch.int32, device=self.device)
        self.align = B.alloc_align_outputs(T, k, self.E_local, block_size, self.device)
        self.capacity = self.align.capacity
        self.workspace = B.alloc_workspace(T, k, self.E_local, self.device)
        self.dispatch_workspace = B.alloc_dispatch_workspace(T, k, self.E_local, self.device)
        self.permuted = torch.empty((self.capacity, H), dtype=torch.bfloat16, device=self.device)
        self.out = torch.empty((T, H), dtype=torch.bfloat16, device=self.device)
        # device-side inputs for the end-to-end path
        self.logits_dev = torch.empty((T, E), dtype=logits_dtype, device=self.device)
        self.hidden_dev = torch.empty((T, H), dtype=torch.bfloat16, device=self.device)

    # ------------------------------------------------------------------ stages --
    def gate(self, logits: torch.Tensor, stream=None):
        return B.moe_topk_softmax(logits, self.k, self.renormalize, self.topk_weights, self.topk_ids, stream,
                                  scoring=self.scoring)

    def align_permute(self, topk_ids: Optional[torch.Tensor] = None, stream=None) -> B.AlignResult:
        ids = self.topk_ids if topk_ids is None else topk_ids
        return B.moe_align_permute(ids, self.E, self.block_size, self.expert_map, self.E_local, self.align,
                                   self.workspace, stream)

    def gather(self, hidden: torch.Tensor, stream=None, hidden_ready: bool = False) -> torch.Tensor:
        return B.moe_gather(hidden, self.k, self.align.inv_perm, self.capacity, permuted=self.permuted,
                            device_status=self.workspace, stream=stream, hidden_ready=hidden_ready)

    def combine(self, expert_out: torch.Tensor, topk_weights: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
        w = self.topk_weights if topk_weights is None else topk_weights
        return B.moe_combine(expert_out, w, self.align.inv_perm, self.out, device_status=self.workspace,
                             stream=stream)

    def dispatch(self, logits: Optional[torch.Tensor], hidden: torch.Tensor, stream=None,
                 topk_ids: Optional[torch.Tensor] = None):
        """gate + align + permute-gather through the fused entry point (one kernel for small batches,
        three above).  With ``topk_ids`` given, those routes are aligned instead of gating ``logits``."""
        given = topk_ids is not None
        return B.moe_route_dispatch(None if given else logits, hidden, self.k, self.renormalize, self.block_size,
                                    self.expert_map, self.E_local, None if given else self.topk_weights,
                                    topk_ids if given else self.topk_ids, self.align, self.permuted,
                                    self.dispatch_workspace, stream, given_ids=given, E=self.E,
                                    scoring=self.scoring)

    @property
    def small_batch(self) -> bool:
        """True when moe_route_dispatch runs as a single kernel (decode-sized batches)."""
        return self.T <= 32 and self.T * self.k <= 256 and self.E <= 256

    def step(self, logits: torch.Tensor, hidden: torch.Tensor, expert_out: torch.Tensor, stream=None) -> torch.Tensor:
        """gate + align + permute-gather + combine; expert_out stands in for the expert MLPs' output.

        Runs the fused dispatch (one kernel for decode-sized batches, three above) then the combine;
        it measured faster than the four stage entry points at every size."""
        return self.step_fused(logits, hidden, expert_out, stream)

    def step_staged(self, logits: torch.Tensor, hidden: torch.Tensor, expert_out: torch.Tensor,
                    stream=None) -> torch.Tensor:
        """The step through the four stage entry points."""
        self.gate(logits, stream)
        self.align_permute(stream=stream)
        self.gather(hidden, stream, hidden_ready=True)  # hidden is an input of the step: ready before gating
        return self.combine(expert_out, stream=stream)

    def step_fused(self, logits: torch.Tensor, hidden: torch.Tensor, expert_out: torch.Tensor,
                   stream=None) -> torch.Tensor:
        """The step with gating + align + gather fused into moe_route_dispatch."""
        self.dispatch(logits, hidden, stream)
        return self.combine(expert_out, stream=stream)

    def step_routes(self, topk_ids: torch.Tensor, topk_weights: torch.Tensor, hidden: torch.Tensor,
                    expert_out: torch.Tensor, stream=None) -> torch.Tensor:
        """The step for routes chosen by the caller (no gating): align + permute-gather + combine."""
        self.dispatch(None, hidden, stream, topk_ids=topk_ids)
        return self.combine(expert_out, topk_weights, stream=stream)

    def step_from_host(self, logits_host: torch.Tensor, hidden_host: torch.Tensor, expert_out: torch.Tensor,
                       out_host: torch.Tensor, stream=None) -> torch.Tensor:
        """End to end: H2D copies of the step's inputs, the step, D2H copy of the combined output.

        Host tensors should be pinned for asynchronous copies; the caller synchronises."""
        s = torch.cuda.current_stream() if stream is None else stream
        with torch.cuda.stream(s):
            self.logits_dev.copy_(logits_host, non_blocking=True)
            self.hidden_dev.copy_(hidden_host, non_blocking=True)
            out = self.step(self.logits_dev, self.hidden_dev, expert_out, s)
            out_host.copy_(out, non_blocking=True)
        return out_host

    def device_status(self, stream=None) -> int:
        """Read and reset the device status words of both paths (synchronises); the first error seen."""
        a = B.moe_read_status(self.workspace, stream)
        b = B.moe_read_status(self.dispatch_workspace, stream)
        return a if a != B.MOE_OK else b


class HostStepPipeline:
    """End-to-end routing steps from pinned host buffers, with the copies overlapped.

    Each ``submit`` enqueues one step: the host->device copies of its logits and hidden rows on a copy
    stream, the step (moe_route_dispatch + moe_combine) on a compute stream, and the device->host copy
    of its combined output on a third stream.  ``depth`` sets of device input and output buffers
    rotate, so step i's inputs are copied in while step i-1 runs and step i-2's output is copied out
    (the two copy directions share no engine).  Events order each buffer set's reuse: a set's inputs
    are overwritten only after the step that read them, its output only after that output has been
    copied out.  The router's other device buffers (routes, align outputs, gathered rows) are used by
    the compute stream alone, in step order.  ``expert_out`` stands in for the expert MLPs' output.
    Host output buffers must stay untouched until ``synchronize`` (or the step's own copy) is done."""

    def __init__(self, router: MoeRouter, expert_out: torch.Tensor, depth: int = 2):
        self.r = router
        self.y = expert_out
        self.depth = depth
        dev = router.device
        self.h2d = torch.cuda.Stream(device=dev)
        self.comp = torch.cuda.Stream(device=dev)
        self.d2h = torch.cuda.Stream(device=dev)
        self.logits = [torch.empty_like(router.logits_dev) for _ in range(depth)]
        self.hidden = [torch.empty_like(router.hidden_dev) for _ in range(depth)]
        self.out = [torch.empty_like(router.out) for _ in range(depth)]
        self.in_ready = [torch.cuda.Event() for _ in range(depth)]
        self.in_free = [torch.cuda.Event() for _ in range(depth)]
        self.done = [torch.cuda.Event() for _ in range(depth)]
        self.out_free = [torch.cuda.Event() for _ in range(depth)]
        self.i = 0

    def submit(self, logits_host: torch.Tensor, hidden_host: torch.Tensor, out_host: torch.Tensor) -> None:
        b = self.i % self.depth
        r = self.r
        self.h2d.wait_event(self.in_free[b])  # (no-op before the set's first use)
        with torch.cuda.stream(self.h2d):
            self.logits[b].copy_(logits_host, non_blocking=True)
            self.hidden[b].copy_(hidden_host, non_blocking=True)
            self.in_ready[b].record(self.h2d)
        self.comp.wait_event(self.in_ready[b])
        self.comp.wait_event(self.out_free[b])
        with torch.cuda.stream(self.comp):
            r.dispatch(self.logits[b], self.hidden[b], stream=self.comp)
            B.moe_combine(self.y, r.topk_weights, r.align.inv_perm, self.out[b], device_status=r.workspace,
                          stream=self.comp)
            self.in_free[b].record(self.comp)
            self.done[b].record(self.comp)
        self.d2h.wait_event(self.done[b])
        with torch.cuda.stream(self.d2h):
            out_host.copy_(self.out[b], non_blocking=True)
            self.out_free[b].record(self.d2h)
        self.i += 1

    def synchronize(self) -> None:
        for s in (self.h2d, self.comp, self.d2h):
            s.synchronize()

    def timed(self, submit_one, n: int):
        """Run ``submit_one(i)`` for i < n between two timing events: one on the copy-in stream before the
        first copy, one on the copy-out stream after the last copy (which follows every earlier step).
        Returns the two events, completed."""
        torch.cuda.synchronize(self.r.device)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(self.h2d)
        for i in range(n):
            submit_one(i)
        e1.record(self.d2h)
        self.synchronize()
        return e0, e1
