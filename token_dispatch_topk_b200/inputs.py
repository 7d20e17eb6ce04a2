"""Seeded synthetic inputs for the MoE token-routing workloads.

This module generates inputs only: router logits, hidden activations, stand-in
expert outputs, expert-parallel maps and injected decode route patterns.  It
holds none of the routing arithmetic, and it is the one module that both the
CUDA path's tests/bench and the CPU oracle's tests read.

Recipe (all seeded; seed s defaults to 0):
  * stream s*4+0: router logits, N(0, sigma^2) drawn in fp32 by torch's CPU
    generator, then rounded to the logits dtype (bf16 round-to-nearest-even);
  * stream s*4+1: hidden activations [T, H], N(0,1) in fp32 -> bf16;
  * stream s*4+2: stand-in expert outputs [capacity, H], N(0,1) -> bf16 (these
    replace the expert GEMMs, which sit between gather and combine);
  * stream s*4+3: the Zipf popularity ranking of the experts (a random
    permutation) for the skewed workload.
Zipf skew (popularity of the expert ranked r proportional to r^-s): the log
popularity -s*ln(r) is added to every token's logit for that expert in fp32
before the rounding to bf16, so the softmax prior follows the Zipf law.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int                 # tokens
    E: int                 # experts (global)
    k: int                 # top-k
    H: int                 # hidden size (bf16 activations)
    block_size: int
    renormalize: bool
    logits_dtype: str = "bf16"   # "bf16" or "f32"
    logits_sigma: float = 1.0
    E_local: Optional[int] = None  # experts owned by this expert-parallel rank (None: all, identity map)
    ep_rank: int = 0
    zipf_s: Optional[float] = None
    description: str = ""

    @property
    def experts_local(self) -> int:
        return self.E if self.E_local is None else self.E_local

    @property
    def capacity(self) -> int:
        """Rows of the block-padded expert-grouped layout (worst case over routings)."""
        return self.T * self.k + self.experts_local * (self.block_size - 1)

    def as_config(self) -> dict:
        d = dataclasses.asdict(self)
        d["E_local"] = self.experts_local
        return d


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny_T64_E8_k2", T=64, E=8, k=2, H=256, block_size=16, renormalize=True,
                 description="tiny: bf16 logits N(0,1), H=256, identity map"),
        Workload("qwen3moe_prefill_T4096_E128_k8", T=4096, E=128, k=8, H=2048, block_size=64, renormalize=True,
                 description="Qwen3-MoE-like prefill: bf16 logits N(0,1), H=2048, identity map"),
        Workload("ep_decode_T2_E160_local40_k6", T=2, E=160, k=6, H=4096, block_size=8, renormalize=True,
                 E_local=40, ep_rank=1,
                 description="DeepSeek-style expert-parallel decode, M=2: rank 1 of 4 owns experts 40..79"),
        Workload("nonpow2_T16384_E60_k4", T=16384, E=60, k=4, H=2048, block_size=64, renormalize=False,
                 logits_dtype="f32", logits_sigma=math.sqrt(2.0),
                 description="non-power-of-2 experts: fp32 logits N(0,2) (variance 2), no renormalisation"),
        Workload("zipf_prefill_T65536_E256_k8_H7168", T=65536, E=256, k=8, H=7168, block_size=128,
                 renormalize=True, zipf_s=1.1,
                 description="large skewed prefill: bf16 logits N(0,1) + Zipf(1.1) expert popularity bias"),
    ]
}

DEFAULT_WORKLOAD = "qwen3moe_prefill_T4096_E128_k8"

# Injected route patterns for the M=2, top-k 6 expert-parallel decode (rank 1 of 4 owns globals 40..79).
# Same experts, disjoint experts, cross-row overlap, twelve distinct local routes and a valid all-remote
# rank, plus within-row duplicates and all duplicates.
DECODE_PATTERNS: Dict[str, List[List[int]]] = {
    "same": [[44, 3, 61, 120, 77, 15], [44, 3, 61, 120, 77, 15]],
    "disjoint": [[44, 3, 61, 120, 77, 15], [52, 90, 70, 8, 45, 150]],
    "cross_row": [[44, 3, 61, 120, 77, 15], [61, 44, 58, 3, 99, 133]],
    "twelve_local": [[40, 47, 54, 61, 68, 75], [43, 50, 57, 64, 71, 79]],
    "all_remote": [[0, 7, 19, 33, 39, 80], [81, 100, 120, 140, 150, 159]],
    "within_row_dup": [[44, 44, 61, 3, 77, 15], [52, 52, 52, 8, 45, 150]],
    "all_duplicate": [[44, 44, 44, 44, 44, 44], [44, 44, 44, 44, 44, 44]],
}


def _gen(seed: int, stream: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 4 + stream)
    return g


def expert_map(wl: Workload) -> Optional[torch.Tensor]:
    """int32 [E] global -> local expert map of the workload's rank (contiguous blocks), or None (identity)."""
    if wl.E_local is None:
        return None
    m = torch.full((wl.E,), -1, dtype=torch.int32)
    lo = wl.ep_rank * wl.E_local
    m[lo:lo + wl.E_local] = torch.arange(wl.E_local, dtype=torch.int32)
    return m


def strided_expert_map(E: int, ranks: int, rank: int) -> torch.Tensor:
    """int32 [E] map for a rank that owns every expert g with g % ranks == rank (local id g // ranks)."""
    g = torch.arange(E, dtype=torch.int32)
    return torch.where(g % ranks == rank, g // ranks, torch.full_like(g, -1)).to(torch.int32)


def zipf_bias(wl: Workload, seed: int = 0) -> Optional[torch.Tensor]:
    """fp32 [E] log-popularity per expert: -s * ln(rank), ranks from a seeded permutation (1 = hottest)."""
    if wl.zipf_s is None:
        return None
    perm = torch.randperm(wl.E, generator=_gen(seed, 3))
    rank = (perm + 1).to(torch.float64)
    return (-wl.zipf_s * torch.log(rank)).to(torch.float32)


def make_logits(wl: Workload, seed: int = 0, T: Optional[int] = None) -> torch.Tensor:
    """Router logits [T, E] on the CPU, bf16 or fp32."""
    T = wl.T if T is None else T
    z = torch.randn((T, wl.E), generator=_gen(seed, 0), dtype=torch.float32)
    if wl.logits_sigma != 1.0:
        z = z * torch.tensor(wl.logits_sigma, dtype=torch.float32)
    b = zipf_bias(wl, seed)
    if b is not None:
        z = z + b[None, :]
    return z.to(torch.bfloat16) if wl.logits_dtype == "bf16" else z


def make_hidden(wl: Workload, seed: int = 0, T: Optional[int] = None, H: Optional[int] = None) -> torch.Tensor:
    """Hidden activations [T, H] bf16 on the CPU."""
    T = wl.T if T is None else T
    H = wl.H if H is None else H
    return torch.randn((T, H), generator=_gen(seed, 1), dtype=torch.float32).to(torch.bfloat16)


def make_expert_out(rows: int, H: int, seed: int = 0, device="cpu", chunk_rows: int = 1 << 16) -> torch.Tensor:
    """Stand-in expert outputs [rows, H] bf16 ~ N(0,1), generated on ``device`` in row chunks.

    On a CUDA device this uses torch's CUDA generator (values differ from the CPU stream of the same seed);
    readers that need the values on the host copy the rows they need back."""
    out = torch.empty((rows, H), dtype=torch.bfloat16, device=device)
    g = _gen(seed, 2, device=device)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        out[r0:r1] = torch.randn((r1 - r0, H), generator=g, dtype=torch.float32, device=device).to(torch.bfloat16)
    return out


def decode_pattern_ids(name: str) -> torch.Tensor:
    return torch.tensor(DECODE_PATTERNS[name], dtype=torch.int32)


def decode_pattern_weights(seed: int = 0, T: int = 2, k: int = 6) -> torch.Tensor:
    """fp32 [T, k] combine weights for injected decode patterns: uniform(0,1) draws (combine is linear in them)."""
    return torch.rand((T, k), generator=_gen(seed, 3), dtype=torch.float32)
