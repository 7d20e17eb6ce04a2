"""GPU parity of the expert-parallel exchange (moe_reduce_partials, and the reduce-scatter form built
from moe_combine and moe_reduce_partials in token_dispatch_topk_b200.dist) against the CPU oracle.

The ranks of an expert-parallel layer run here on one GPU, one after another: each rank's combine
writes each owner's token range into a local buffer standing in for that owner's receive buffer
(on several GPUs, peer memory written over NVLink by the same stores), then every owner reduces its
buffers.  Bars: the reduce bit-exact against the oracle on the same partials; the partial combines
within one bf16 ulp of the oracle's (bit-exact in practice).
"""
import numpy as np
import pytest
import torch

import oracle
import token_dispatch_topk_b200 as tdt
from token_dispatch_topk_b200 import dist as D

from gpu_helpers import COMBINE_MAX_ULP, bf16_bits, bits_to_bf16, require_gpu, ulp_distance_bf16

pytestmark = pytest.mark.gpu


def _partials(n, rows, H, seed):
    """bf16 partials with mixed magnitudes, exact cancellations and signed zeros."""
    rng = np.random.default_rng(seed)
    mags = np.float32(2.0) ** rng.integers(-14, 15, size=(n, rows, H)).astype(np.float32)
    x = (rng.standard_normal((n, rows, H)).astype(np.float32) * mags)
    bits = (x.view(np.uint32) + 0x7FFF + ((x.view(np.uint32) >> 16) & 1)) >> 16
    bits = bits.astype(np.uint16)
    if n >= 2 and rows:
        bits[1, 0] = bits[0, 0] ^ 0x8000        # rank 1 cancels rank 0 in row 0
        bits[:, -1, :2] = 0x8000                # -0 from every rank
    return bits


@pytest.mark.parametrize("n,rows,H", [(1, 5, 8), (2, 37, 264), (3, 64, 2048), (5, 129, 40), (8, 4097, 256),
                                      (16, 33, 16), (4, 0, 64)])
def test_reduce_partials_parity(n, rows, H):
    dev = require_gpu()
    bits = _partials(n, rows, H, seed=n * 1000 + rows + H)
    parts = [bits_to_bf16(bits[r]).to(dev) for r in range(n)]
    out = tdt.moe_reduce_partials(parts)
    torch.cuda.synchronize()
    ref = oracle.reduce_partials(bits) if rows else np.zeros((0, H), np.uint16)
    assert np.array_equal(bf16_bits(out), ref), np.nonzero(bf16_bits(out) != ref)
    if rows:  # in place: out may be the first partial
        tdt.moe_reduce_partials(parts, out=parts[0])
        torch.cuda.synchronize()
        assert np.array_equal(bf16_bits(parts[0]), ref)


def test_reduce_partials_errors():
    dev = require_gpu()
    parts = [torch.zeros((4, 8), dtype=torch.bfloat16, device=dev) for _ in range(17)]
    with pytest.raises(tdt.MoeError) as e:
        tdt.moe_reduce_partials(parts)
    assert e.value.status == tdt.MOE_ERR_UNSUPPORTED
    flat = torch.zeros(4 * 8 + 1, dtype=torch.bfloat16, device=dev)
    misaligned = flat[1:].view(4, 8)  # 2 bytes past a 16-byte boundary
    with pytest.raises(tdt.MoeError) as e:
        tdt.moe_reduce_partials([parts[0], misaligned])
    assert e.value.status == tdt.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("T,E,k,H,bs,world", [(300, 64, 8, 256, 16, 4), (2, 160, 6, 4096, 8, 4), (97, 60, 4, 64, 8, 3)],
                         ids=["prefill_like", "decode_T2_owners_without_tokens", "nonpow2_three_ranks"])
def test_expert_parallel_reduce_scatter_emulated(T, E, k, H, bs, world):
    """Each rank: align with its expert_map (routes from the oracle's gating), its own expert outputs,
    its combine written per owner into the owners' receive buffers; each owner: moe_reduce_partials.
    The concatenated owner outputs equal the oracle's reduce of the GPU's partials, bit for bit, and
    the GPU partials are within one bf16 ulp of the oracle's partial combines."""
    dev = require_gpu()
    rng = np.random.default_rng(T + E + world)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    w_ref, ids_ref = oracle.topk_softmax(logits, k, True)
    w = torch.from_numpy(w_ref).to(dev)
    ids = torch.from_numpy(ids_ref).to(dev)
    ranges = [D.ep_token_range(T, world, o) for o in range(world)]
    # receive buffers: owner o holds one [hi - lo, H] slot per rank
    recv = [torch.full((world, hi - lo, H), -1.0, dtype=torch.bfloat16, device=dev) for lo, hi in ranges]
    partial_bits = []
    for r in range(world):
        emap, El = D.ep_expert_map(E, world, r)
        al = tdt.moe_align_permute(ids, E, bs, emap.to(dev), El)
        y_bits = (rng.standard_normal((al.capacity, H)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
        y = bits_to_bf16(y_bits).to(dev)
        D.ep_combine_to_owners(y, w, al.inv_perm, [recv[o][r] for o in range(world)])
        torch.cuda.synchronize()
        # this rank's whole partial, as written into the owners' buffers
        got = np.concatenate([bf16_bits(recv[o][r]) for o in range(world)]) if T else np.zeros((0, H), np.uint16)
        al_ref = oracle.align_permute(ids_ref, E, bs, emap.numpy(), El)
        ref = oracle.combine(y_bits, w_ref, al_ref["inv_perm"])
        assert (ulp_distance_bf16(got, ref) <= COMBINE_MAX_ULP).all(), r
        partial_bits.append(got)
    outs = []
    for o, (lo, hi) in enumerate(ranges):
        if hi > lo:
            outs.append(bf16_bits(D.ep_reduce_received([recv[o][r] for r in range(world)])))
    torch.cuda.synchronize()
    got = np.concatenate(outs)
    assert np.array_equal(got, oracle.reduce_partials(np.stack(partial_bits)))
