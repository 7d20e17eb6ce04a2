"""GPU parity of the fused dispatch (moe_route_dispatch: gating + align + permute-gather) against
the CPU oracle pipeline, through the C ABI.

Two kernel paths sit behind the call: one kernel with one CTA per slot for small batches
(T <= 32, T*k <= 256 and E <= 256) and the tiled three-kernel path above that.  Shapes cover both sides of every
one of those limits, one and many gating tiles with a ragged last tile, maps with remote and
out-of-range values, every gating vector width, k up to 32, 1024 experts, T = 0 and the decode size,
with logits-derived routes and with routes given by the caller.  Bars as for the stage entry points:
ids, align outputs and gathered rows bit-exact, weights within 2e-6.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import token_dispatch_topk_b200 as tdt
from token_dispatch_topk_b200 import inputs as I

from gpu_helpers import TOPK_WEIGHT_ATOL, assert_align_equal, bf16_bits, logits_for_oracle, np_i32, require_gpu

pytestmark = pytest.mark.gpu

CASES = [
    # name, T, E, k, dtype, renorm, map kind, E_local, bs, H
    ("tiny", 64, 8, 2, torch.bfloat16, True, None, 8, 16, 256),
    ("prefill_ragged", 4100, 128, 8, torch.bfloat16, True, None, 128, 64, 2048),
    ("decode_rank1", 2, 160, 6, torch.bfloat16, True, "rank1", 40, 8, 4096),
    ("nonpow2_fp32", 3000, 60, 4, torch.float32, False, None, 60, 64, 264),
    ("strided_map", 777, 160, 6, torch.bfloat16, True, "strided", 40, 8, 512),
    ("bad_map_values", 500, 64, 4, torch.bfloat16, True, "bad", 16, 16, 64),
    ("k32_fp32", 300, 64, 32, torch.float32, True, None, 64, 8, 128),
    ("wide_1024", 257, 1024, 8, torch.bfloat16, False, None, 1024, 4, 128),
    ("odd_e_bf16", 333, 61, 5, torch.bfloat16, True, None, 61, 3, 16),
    ("many_tiles_small_bs", 9000, 32, 2, torch.bfloat16, True, None, 32, 1, 8),
    ("zero_tokens", 0, 16, 4, torch.bfloat16, True, None, 16, 8, 64),
    # single-kernel path (one CTA per slot) and its limits
    ("small_T1", 1, 64, 4, torch.bfloat16, True, None, 64, 16, 512),
    ("small_T32_k8_fp32", 32, 64, 8, torch.float32, True, None, 64, 8, 128),
    ("tile_T32_k9", 32, 64, 9, torch.bfloat16, True, None, 64, 8, 128),
    ("tile_T9_k32_fp32", 9, 64, 32, torch.float32, True, None, 64, 8, 64),
    ("small_T8_k32", 8, 64, 32, torch.bfloat16, False, None, 64, 4, 64),
    ("tile_small_T_wide_1024_fp32", 8, 1024, 8, torch.float32, False, None, 1024, 4, 64),
    ("tile_small_T_wide_1024_bf16_map", 5, 1024, 8, torch.bfloat16, True, "strided", 256, 2, 64),
    ("small_E256_fp32", 8, 256, 8, torch.float32, False, None, 256, 4, 64),
    ("small_E256_bf16_map", 5, 256, 8, torch.bfloat16, True, "strided", 64, 2, 64),
    ("tile_E257", 4, 257, 8, torch.bfloat16, True, None, 257, 4, 64),
    ("small_bad_map_values", 20, 64, 4, torch.bfloat16, True, "bad", 16, 16, 64),
    ("small_odd_e_fp32", 31, 61, 5, torch.float32, True, None, 61, 3, 16),
    ("small_long_rows", 3, 32, 2, torch.bfloat16, True, None, 32, 4, 65536),
    ("small_rows_past_prefetch", 2, 160, 6, torch.bfloat16, True, "rank1", 40, 8, 8200),
    ("tile_T33_decode_map", 33, 160, 6, torch.bfloat16, True, "rank1", 40, 8, 4096),
    # degenerate shapes on both paths
    ("tile_k1_bs1_H8", 100, 16, 1, torch.bfloat16, True, None, 16, 1, 8),
    ("tile_one_local_expert", 200, 32, 4, torch.bfloat16, True, "one_local", 1, 8, 64),
    ("small_one_local_expert", 3, 32, 4, torch.float32, False, "one_local", 1, 8, 64),
    ("small_k1_bs1_H8", 1, 4, 1, torch.bfloat16, False, None, 4, 1, 8),
    ("tile_all_remote", 64, 32, 4, torch.bfloat16, True, "none_local", 8, 16, 32),
    # one thread per row (T >= 1024, E <= 64 in whole 16-byte chunks, k <= 8): maps, ties, k == E,
    # ragged last tiles
    ("lanes_bf16_E64_k8_strided_map", 1500, 64, 8, torch.bfloat16, True, "strided", 16, 16, 64),
    ("lanes_fp32_E8_k8_k_equals_E", 1100, 8, 8, torch.float32, False, None, 8, 4, 32),
    ("lanes_bf16_E16_k1_ties", 2049, 16, 1, torch.bfloat16, True, None, 16, 8, 16),
    ("lanes_fp32_E12_k3_one_local", 1030, 12, 3, torch.float32, True, "one_local", 1, 2, 16),
    ("lanes_bf16_bad_map_values", 1200, 64, 4, torch.bfloat16, True, "bad", 16, 16, 64),
    ("lanes_fp32_E48_k6_ties", 2077, 48, 6, torch.float32, False, None, 48, 32, 48),
    ("lanes_bf16_E64_k8_ties", 2100, 64, 8, torch.bfloat16, True, None, 64, 64, 64),
    ("lanes_bf16_E56_k7_strided_map", 1111, 56, 7, torch.bfloat16, False, "strided", 14, 16, 32),
    ("lanes_wide_bf16_E256_k8_strided_map", 16500, 256, 8, torch.bfloat16, True, "strided", 64, 128, 16),
    ("lanes_wide_bf16_E192_k5_ties", 16401, 192, 5, torch.bfloat16, False, None, 192, 32, 8),
    # more tiles than the gating kernel's CTAs resident at once (625 tiles of 512 threads); many local
    # experts (a long tile scan per expert); ragged lanes batches
    ("many_tiles_fp32_E128", 20000, 128, 8, torch.float32, True, None, 128, 16, 16),
    ("many_tiles_E512", 5000, 512, 8, torch.bfloat16, True, None, 512, 16, 64),
    ("lanes_fp32_E60_ragged", 16400, 60, 4, torch.float32, False, None, 60, 64, 16),
    ("lanes_bf16_E61_no_lanes_odd", 4000, 61, 3, torch.bfloat16, True, None, 61, 5, 16),
]


def _map(kind, E, E_local):
    if kind is None:
        return None
    if kind == "rank1":
        m = np.full(E, -1, np.int32)
        m[E_local:2 * E_local] = np.arange(E_local)
        return m
    if kind == "strided":
        return I.strided_expert_map(E, 4, 1).numpy()
    if kind == "one_local":  # a single local expert: global 5
        m = np.full(E, -1, np.int32)
        m[5] = 0
        return m
    if kind == "none_local":  # a rank whose experts the router never picks (map covers only the last 8)
        m = np.full(E, -1, np.int32)
        m[E - E_local:] = np.arange(E_local)
        return m
    if kind == "bad":  # some globals map past E_local or below -1: those slots are dropped and flagged
        m = np.full(E, -1, np.int32)
        m[:E_local] = np.arange(E_local)
        m[E_local] = E_local + 3
        m[E_local + 1] = -5
        return m
    raise ValueError(kind)


@pytest.mark.parametrize("name,T,E,k,dtype,renorm,kind,E_local,bs,H", CASES, ids=[c[0] for c in CASES])
def test_dispatch_parity(name, T, E, k, dtype, renorm, kind, E_local, bs, H):
    dev = require_gpu()
    g = torch.Generator().manual_seed(T + 7 * E + k)
    x = torch.randn((T, E), generator=g).to(dtype)
    if name.endswith("_ties"):  # integer logits: equal values at the k boundary in most rows
        x = torch.randint(0, 4, (T, E), generator=g).to(dtype)
    if kind == "none_local":  # the last E_local experts never make the top k
        x[:, E - E_local:] -= 50.0
    if kind == "bad":  # make the flagged globals win often
        x[:, E_local] += 3.0
        x[:, E_local + 1] += 3.0
    hidden = torch.randn((T, H), generator=g).to(torch.bfloat16)
    emap = _map(kind, E, E_local)
    emap_d = None if emap is None else torch.from_numpy(emap).to(dev)
    ws = tdt.alloc_dispatch_workspace(T, k, E_local, dev)
    w_ref, ids_ref = oracle.topk_softmax(logits_for_oracle(x), k, renorm)
    al = oracle.align_permute(ids_ref, E, bs, emap, E_local)
    npad = int(al["num_tokens_post_pad"][0])
    perm_ref = oracle.gather(bf16_bits(hidden), k, al["sorted_token_ids"], npad, al["capacity"])
    real = al["sorted_token_ids"][:npad] != T * k
    for call in range(2):  # the second call checks that the workspace was left ready
        w, ids, align, perm = tdt.moe_route_dispatch(x.to(dev), hidden.to(dev), k, renorm, bs, emap_d, E_local,
                                                     workspace=ws)
        torch.cuda.synchronize()
        assert np.array_equal(np_i32(ids), ids_ref), (name, call)
        if T:
            assert np.abs(w.cpu().numpy() - w_ref).max() <= TOPK_WEIGHT_ATOL, (name, call)
        assert_align_equal(align, al, f"{name} call {call}")
        assert np.array_equal(bf16_bits(perm[:npad])[real], perm_ref[:npad][real]), (name, call)
        status = tdt.moe_read_status(ws)
        assert status == (tdt.MOE_ERR_BAD_EXPERT_ID if kind == "bad" else tdt.MOE_OK), (name, status)


@pytest.mark.parametrize("workload", ["qwen3moe_prefill_T4096_E128_k8", "nonpow2_T16384_E60_k4",
                                      "zipf_prefill_T65536_E256_k8_H7168"])
def test_dispatch_matches_stage_entry_points(workload):
    """The fused dispatch and the three stage calls it replaces give identical outputs (one warp per
    row on the prefill workload, lanes per row on the non-power-of-2 and skewed ones)."""
    dev = require_gpu()
    wl = I.WORKLOADS[workload]
    logits, hidden = I.make_logits(wl, device=dev), I.make_hidden(wl, device=dev)
    a = tdt.MoeRouter(wl.T, wl.E, wl.k, wl.H, wl.block_size, wl.renormalize, logits_dtype=logits.dtype, device=dev)
    b = tdt.MoeRouter(wl.T, wl.E, wl.k, wl.H, wl.block_size, wl.renormalize, logits_dtype=logits.dtype, device=dev)
    a.dispatch(logits, hidden)
    b.gate(logits)
    b.align_permute()
    b.gather(hidden)
    torch.cuda.synchronize()
    for name in ("counts", "offsets", "sorted_token_ids", "expert_ids", "num_tokens_post_pad", "inv_perm"):
        assert torch.equal(getattr(a.align, name), getattr(b.align, name)), name
    assert torch.equal(a.topk_ids, b.topk_ids) and torch.equal(a.topk_weights, b.topk_weights)
    npad = int(a.align.num_tokens_post_pad.item())
    real = (a.align.sorted_token_ids[:npad] != wl.T * wl.k)
    assert torch.equal(a.permuted[:npad][real], b.permuted[:npad][real])


GIVEN = [
    # name, T, k, E, map kind, E_local, bs, H
    ("small_decode_patterns", 2, 6, 160, "rank1", 40, 8, 4096),
    ("tile_decode_patterns_tiled", 70, 6, 160, "rank1", 40, 8, 256),
]


@pytest.mark.parametrize("name,T,k,E,kind,E_local,bs,H", GIVEN, ids=[c[0] for c in GIVEN])
def test_dispatch_given_routes(name, T, k, E, kind, E_local, bs, H):
    """MOE_DISPATCH_GIVEN_IDS: every injected decode route pattern (rows repeated to T), plus a
    pattern with out-of-range ids, through the small and the tiled path; topk_weights untouched."""
    dev = require_gpu()
    emap = _map(kind, E, E_local)
    emap_d = torch.from_numpy(emap).to(dev)
    hidden = torch.randn((T, H), generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    ws = tdt.alloc_dispatch_workspace(T, k, E_local, dev)
    patterns = dict(I.DECODE_PATTERNS)
    patterns["out_of_range"] = [[44, -1, 160, 3, 1000, 61], [-7, 44, 52, 52, 159, 0]]
    for pname, rows in patterns.items():
        ids = np.array([rows[t % 2] for t in range(T)], np.int32)
        al = oracle.align_permute(ids, E, bs, emap, E_local)
        npad = int(al["num_tokens_post_pad"][0])
        perm_ref = oracle.gather(bf16_bits(hidden), k, al["sorted_token_ids"], npad, al["capacity"])
        real = al["sorted_token_ids"][:npad] != T * k
        sentinel = torch.full((T, k), -2.5, dtype=torch.float32, device=dev)
        _, _, align, perm = tdt.moe_route_dispatch(None, hidden.to(dev), k, True, bs, emap_d, E_local,
                                                   topk_weights=sentinel, topk_ids=torch.from_numpy(ids).to(dev),
                                                   workspace=ws, given_ids=True, E=E)
        torch.cuda.synchronize()
        assert_align_equal(align, al, f"{name}/{pname}")
        assert np.array_equal(bf16_bits(perm[:npad])[real], perm_ref[:npad][real]), (name, pname)
        assert bool((sentinel == -2.5).all()), (name, pname)
        status = tdt.moe_read_status(ws)
        assert status == (tdt.MOE_ERR_BAD_EXPERT_ID if pname == "out_of_range" else tdt.MOE_OK), (name, pname)


@pytest.mark.parametrize("T,E,k,dtype,renorm,E_local,bs,H", [
    (2, 160, 6, torch.bfloat16, True, 160, 8, 512),       # single-kernel path
    (20, 64, 4, torch.float32, False, 64, 16, 64),
    (300, 128, 8, torch.bfloat16, True, 128, 64, 256),    # three-kernel path
    (777, 60, 4, torch.float32, False, 60, 64, 128),
    (2500, 60, 4, torch.float32, True, 60, 64, 128),     # one thread per row
    (1300, 64, 8, torch.bfloat16, False, 64, 16, 64),
], ids=["small_bf16", "small_fp32", "tile_bf16", "tile_fp32", "lanes_fp32", "lanes_bf16"])
def test_dispatch_sigmoid_scoring(T, E, k, dtype, renorm, E_local, bs, H):
    """moe_route_dispatch with MOE_SCORING_SIGMOID: weights from the sigmoid reading, the rest as for softmax."""
    dev = require_gpu()
    g = torch.Generator().manual_seed(T * 13 + E)
    x = torch.randn((T, E), generator=g).to(dtype)
    hidden = torch.randn((T, H), generator=g).to(torch.bfloat16)
    w_ref, ids_ref = oracle.topk_sigmoid(logits_for_oracle(x), k, renorm)
    al = oracle.align_permute(ids_ref, E, bs)
    npad = int(al["num_tokens_post_pad"][0])
    perm_ref = oracle.gather(bf16_bits(hidden), k, al["sorted_token_ids"], npad, al["capacity"])
    real = al["sorted_token_ids"][:npad] != T * k
    w, ids, align, perm = tdt.moe_route_dispatch(x.to(dev), hidden.to(dev), k, renorm, bs, scoring="sigmoid")
    torch.cuda.synchronize()
    assert np.array_equal(np_i32(ids), ids_ref)
    assert np.abs(w.cpu().numpy() - w_ref).max() <= TOPK_WEIGHT_ATOL
    assert_align_equal(align, al, "sigmoid dispatch")
    assert np.array_equal(bf16_bits(perm[:npad])[real], perm_ref[:npad][real])


def test_dispatch_workspace_shared_across_sizes():
    """One workspace, large enough for every call, used by calls of different sizes and tile layouts:
    each call is correct whatever the previous one left in the workspace."""
    dev = require_gpu()
    shapes = [(3000, 60, 4, 60), (5000, 512, 8, 512), (3000, 60, 4, 60), (700, 128, 8, 128), (5000, 512, 8, 512),
              (700, 128, 8, 128)]
    nbytes = max(tdt.moe_route_dispatch_workspace_bytes(T, k, El) for T, _, k, El in shapes)
    ws = torch.zeros((nbytes + 3) // 4, dtype=torch.int32, device=dev)
    for i, (T, E, k, El) in enumerate(shapes):
        g = torch.Generator().manual_seed(100 + i)
        x = torch.randn((T, E), generator=g).to(torch.bfloat16)
        hidden = torch.randn((T, 16), generator=g).to(torch.bfloat16)
        w_ref, ids_ref = oracle.topk_softmax(bf16_bits(x), k, True)
        al = oracle.align_permute(ids_ref, E, 16)
        _, ids, align, _ = tdt.moe_route_dispatch(x.to(dev), hidden.to(dev), k, True, 16, workspace=ws)
        torch.cuda.synchronize()
        assert np.array_equal(np_i32(ids), ids_ref), i
        assert_align_equal(align, al, f"call {i}: T={T} E={E}")
        assert tdt.moe_read_status(ws) == tdt.MOE_OK, i
