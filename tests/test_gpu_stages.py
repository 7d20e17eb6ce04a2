"""GPU parity, stage by stage, against the CPU oracle through the C ABI.

Each stage is fed the oracle's own upstream outputs, so a mismatch points at one kernel.
Shapes cover every vector width of the gating kernel, one and many align tiles with a
ragged last tile, maps with remote and out-of-range ids, and gather/combine rows with
ragged 16-byte chunk counts.  Bars: ids, counts, offsets, sorted ids, expert ids, N_pad,
inv_perm and gathered rows bit-exact; gating weights within 2e-6; combine within 1 bf16 ulp.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import token_dispatch_topk_b200 as tdt
from token_dispatch_topk_b200 import inputs as I

from gpu_helpers import (COMBINE_MAX_ULP, TOPK_WEIGHT_ATOL, assert_align_equal, bf16_bits, bits_to_bf16,
                         logits_for_oracle, np_i32, require_gpu, ulp_distance_bf16)

pytestmark = pytest.mark.gpu


def _logits(T, E, dtype, sigma=1.0, seed=0, ties=False):
    g = torch.Generator().manual_seed(1000 + seed)
    if ties:
        x = torch.randint(0, 4, (T, E), generator=g).float()
    else:
        x = torch.randn((T, E), generator=g) * sigma
    return x.to(dtype)


TOPK_CASES = [
    # T, E, k, dtype, renormalize, sigma, ties
    (64, 8, 2, torch.bfloat16, True, 1.0, False),
    (4096, 128, 8, torch.bfloat16, True, 1.0, False),
    (2, 160, 6, torch.bfloat16, True, 1.0, False),
    (2000, 60, 4, torch.float32, False, math.sqrt(2.0), False),
    (3000, 256, 8, torch.bfloat16, True, 1.0, False),
    (1, 1, 1, torch.bfloat16, False, 1.0, False),
    (5, 2, 2, torch.float32, True, 1.0, False),
    (37, 7, 3, torch.bfloat16, True, 1.0, False),          # 14-byte rows: scalar loads
    (129, 60, 4, torch.bfloat16, False, 1.0, False),       # 120-byte rows: 8-byte loads
    (100, 61, 5, torch.bfloat16, True, 1.0, False),        # odd E: scalar loads
    (77, 33, 32, torch.float32, True, 1.0, False),         # k = 32
    (50, 1024, 32, torch.bfloat16, False, 1.0, False),     # E = 1024: 4 chunks per lane
    (50, 1000, 8, torch.float32, True, 3.0, False),        # 8 chunks of 4 per lane
    (50, 1023, 7, torch.float32, False, 1.0, False),       # scalar, 32 per lane
    (999, 128, 8, torch.bfloat16, True, 1.0, True),        # tie-heavy: integer logits
    (999, 256, 8, torch.bfloat16, False, 1.0, True),
    (333, 8, 8, torch.bfloat16, True, 1.0, True),          # k == E
    # one thread per row (T >= 1024, E <= 64 in whole 16-byte chunks, k <= 8)
    (1500, 64, 8, torch.bfloat16, True, 1.0, True),        # tie-heavy
    (1024, 32, 1, torch.float32, False, 1.0, False),
    (4097, 16, 2, torch.bfloat16, False, 1.0, True),       # ragged last tile, ties
    (2048, 48, 6, torch.float32, True, 2.0, True),
    (1025, 8, 8, torch.bfloat16, True, 1.0, False),        # k == E
    (1100, 60, 7, torch.float32, False, 8.0, False),       # wide logits: tiny weights
    (1500, 64, 8, torch.bfloat16, False, 1.0, True),       # bf16 keys, tie-heavy, full-row denominator
    (2049, 56, 5, torch.bfloat16, True, 1.0, True),        # ragged last tile, ties
    (16400, 256, 8, torch.bfloat16, True, 1.0, True),      # wide bf16 rows, eight lanes per row, ties
    (16500, 192, 6, torch.bfloat16, False, 1.0, False),    # wide bf16 rows, three chunks per lane
]


@pytest.mark.parametrize("T,E,k,dtype,renorm,sigma,ties", TOPK_CASES)
def test_topk_softmax_parity(T, E, k, dtype, renorm, sigma, ties):
    dev = require_gpu()
    x = _logits(T, E, dtype, sigma, seed=T + E, ties=ties)
    w, ids = tdt.moe_topk_softmax(x.to(dev), k, renorm)
    torch.cuda.synchronize()
    w_ref, ids_ref = oracle.topk_softmax(logits_for_oracle(x), k, renorm)
    assert np.array_equal(np_i32(ids), ids_ref), np.nonzero(np_i32(ids) != ids_ref)
    err = np.abs(w.cpu().numpy().astype(np.float64) - w_ref.astype(np.float64))
    assert err.max() <= TOPK_WEIGHT_ATOL, err.max()


SIGMOID_CASES = [
    # T, E, k, dtype, renormalize, sigma, ties  (sub-warp rows, one warp per row, fp32, wide, tie-heavy, tails)
    (64, 8, 2, torch.bfloat16, True, 1.0, False),
    (37, 7, 3, torch.float32, False, 1.0, False),
    (4096, 128, 8, torch.bfloat16, True, 1.0, False),
    (2000, 60, 4, torch.float32, False, math.sqrt(2.0), False),
    (2, 160, 6, torch.bfloat16, False, 1.0, False),
    (50, 1000, 8, torch.float32, True, 3.0, False),
    (999, 256, 8, torch.bfloat16, True, 1.0, True),
    (300, 64, 8, torch.float32, False, 30.0, False),       # far tails: scores near 0 and 1
    (1500, 64, 8, torch.bfloat16, True, 1.0, True),        # one thread per row, tie-heavy
    (1100, 24, 3, torch.float32, False, 30.0, False),      # one thread per row, far tails
    (16400, 256, 8, torch.bfloat16, True, 1.0, False),     # wide bf16 rows, eight lanes per row
]


@pytest.mark.parametrize("T,E,k,dtype,renorm,sigma,ties", SIGMOID_CASES)
def test_topk_sigmoid_parity(T, E, k, dtype, renorm, sigma, ties):
    """The sigmoid scoring variant (MOE_SCORING_SIGMOID) against the oracle's reading of it."""
    dev = require_gpu()
    x = _logits(T, E, dtype, sigma, seed=3 * T + E, ties=ties)
    w, ids = tdt.moe_topk_softmax(x.to(dev), k, renorm, scoring="sigmoid")
    torch.cuda.synchronize()
    w_ref, ids_ref = oracle.topk_sigmoid(logits_for_oracle(x), k, renorm)
    assert np.array_equal(np_i32(ids), ids_ref), np.nonzero(np_i32(ids) != ids_ref)
    err = np.abs(w.cpu().numpy().astype(np.float64) - w_ref.astype(np.float64))
    assert err.max() <= TOPK_WEIGHT_ATOL, err.max()


def test_topk_softmax_misaligned_rows():
    """A logits view that starts 2 bytes past a 16-byte boundary takes the narrow-load path."""
    dev = require_gpu()
    T, E, k = 300, 128, 8
    flat = _logits(T * E + 8, 1, torch.bfloat16).reshape(-1)
    x = flat[1:1 + T * E].reshape(T, E)
    xd = flat.to(dev)[1:1 + T * E].reshape(T, E)
    assert xd.data_ptr() % 16 != 0
    w, ids = tdt.moe_topk_softmax(xd, k, True)
    w_ref, ids_ref = oracle.topk_softmax(bf16_bits(x), k, True)
    assert np.array_equal(np_i32(ids), ids_ref)
    assert np.abs(w.cpu().numpy() - w_ref).max() <= TOPK_WEIGHT_ATOL


def _ids_random(T, k, E, seed, lo=0, hi=None):
    g = np.random.default_rng(seed)
    hi = E if hi is None else hi
    return g.integers(lo, hi, size=(T, k)).astype(np.int32)


ALIGN_CASES = [
    # name, T, k, E_global, map kind, E_local, block_size
    ("tiny", 64, 2, 8, None, 8, 16),
    ("prefill", 4096, 8, 128, None, 128, 64),
    ("nonpow2", 16384, 4, 60, None, 60, 64),
    ("ragged_tail", 5001, 3, 64, None, 64, 16),
    ("empty", 0, 4, 16, None, 16, 8),
    ("one_slot", 1, 1, 1, None, 1, 1),
    ("bs1_wide", 513, 8, 1024, None, 1024, 1),
    ("wide_multi_tile", 3000, 8, 1024, None, 1024, 32),
    ("strided_map_multi_tile", 3000, 6, 160, "strided", 40, 8),
    ("rank_map_single_tile", 300, 6, 160, "rank1", 40, 8),
    ("bad_ids_multi_tile", 2500, 4, 100, "rank1_bad", 25, 16),
    ("all_remote_multi_tile", 1000, 8, 160, "none_local", 40, 8),
    ("one_hot_expert", 3000, 2, 64, "hot", 64, 64),
]


def _map_and_ids(kind, T, k, E, E_local, seed):
    if kind is None:
        return None, _ids_random(T, k, E, seed)
    if kind == "strided":
        return I.strided_expert_map(E, 4, 1).numpy(), _ids_random(T, k, E, seed)
    if kind == "rank1":
        m = np.full(E, -1, np.int32)
        m[E_local:2 * E_local] = np.arange(E_local)
        return m, _ids_random(T, k, E, seed)
    if kind == "rank1_bad":
        m = np.full(E, -1, np.int32)
        m[E_local:2 * E_local] = np.arange(E_local)
        return m, _ids_random(T, k, E, seed, lo=-3, hi=E + 3)
    if kind == "none_local":
        m = np.full(E, -1, np.int32)
        m[E_local:2 * E_local] = np.arange(E_local)
        ids = _ids_random(T, k, E, seed)
        ids[(ids >= E_local) & (ids < 2 * E_local)] = 0
        return m, ids
    if kind == "hot":
        ids = _ids_random(T, k, E, seed)
        ids[:, 0] = 17
        ids[: T // 2, 1] = 17
        return None, ids
    raise ValueError(kind)


@pytest.mark.parametrize("name,T,k,E,kind,E_local,bs", ALIGN_CASES, ids=[c[0] for c in ALIGN_CASES])
def test_align_permute_parity(name, T, k, E, kind, E_local, bs):
    dev = require_gpu()
    emap, ids = _map_and_ids(kind, T, k, E, E_local, seed=T * 7 + k)
    ref = oracle.align_permute(ids, E, bs, emap, E_local)
    ids_d = torch.from_numpy(ids).to(dev)
    emap_d = None if emap is None else torch.from_numpy(np.ascontiguousarray(emap, np.int32)).to(dev)
    ws = tdt.alloc_workspace(T, k, E_local, dev)
    for rep in range(2):  # the second call checks that the workspace was left ready
        out = tdt.moe_align_permute(ids_d, E, bs, emap_d, E_local, workspace=ws)
        torch.cuda.synchronize()
        assert_align_equal(out, ref, f"{name} call {rep}")
    status = tdt.moe_read_status(ws)
    expect_bad = kind == "rank1_bad"
    assert status == (tdt.MOE_ERR_BAD_EXPERT_ID if expect_bad else tdt.MOE_OK), status
    assert tdt.moe_read_status(ws) == tdt.MOE_OK  # reading resets the word


def test_align_decode_patterns():
    dev = require_gpu()
    wl = I.WORKLOADS["ep_decode_T2_E160_local40_k6"]
    emap = I.expert_map(wl)
    for name in I.DECODE_PATTERNS:
        ids = I.decode_pattern_ids(name)
        ref = oracle.align_permute(ids.numpy(), wl.E, wl.block_size, emap.numpy(), wl.E_local)
        out = tdt.moe_align_permute(ids.to(dev), wl.E, wl.block_size, emap.to(dev), wl.E_local)
        torch.cuda.synchronize()
        assert_align_equal(out, ref, name)


GATHER_CASES = [
    # T, k, E, bs, H
    (64, 2, 8, 16, 256),
    (2, 6, 160, 8, 4096),     # segmented rows
    (300, 8, 128, 64, 2048),
    (257, 4, 60, 64, 264),    # 33 chunks per row: ragged lanes
    (100, 8, 256, 128, 7168),
    (50, 3, 12, 4, 8),        # one chunk per row
]


def _align_for(T, k, E, bs, seed):
    ids = _ids_random(T, k, E, seed)
    return ids, oracle.align_permute(ids, E, bs)


@pytest.mark.parametrize("T,k,E,bs,H", GATHER_CASES)
@pytest.mark.parametrize("zero_pad", [False, True])
def test_gather_parity(T, k, E, bs, H, zero_pad):
    dev = require_gpu()
    ids, ref = _align_for(T, k, E, bs, seed=T + H)
    hidden = I.make_hidden(I.WORKLOADS["tiny_T64_E8_k2"], seed=3, T=T, H=H)
    hb = bf16_bits(hidden)
    npad = int(ref["num_tokens_post_pad"][0])
    C = ref["capacity"]
    fill = 0x7FC1  # a NaN pattern no gather writes
    want = oracle.gather(hb, k, ref["sorted_token_ids"], npad, C, zero_pad=zero_pad, fill=fill)
    perm = bits_to_bf16(np.full((C, H), fill, np.uint16)).to(dev)
    sti = torch.from_numpy(ref["sorted_token_ids"]).to(dev)
    np_d = torch.from_numpy(ref["num_tokens_post_pad"]).to(dev)
    inv = torch.from_numpy(ref["inv_perm"]).to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    tdt.moe_gather(hidden.to(dev), k, inv, C, sti, np_d, zero_pad=zero_pad, permuted=perm, device_status=status)
    got = bf16_bits(perm)
    bad = np.nonzero((got != want).any(1))[0]
    assert bad.size == 0, f"rows differ: {bad[:10]}"
    assert tdt.moe_read_status(status) == tdt.MOE_OK


COMBINE_CASES = [
    # T, k, E, bs, H, renorm
    (64, 2, 8, 16, 256, True),
    (2, 6, 160, 8, 4096, True),
    (300, 8, 128, 64, 2048, True),
    (257, 4, 60, 64, 264, False),
    (100, 8, 256, 128, 7168, True),
    (77, 32, 64, 8, 64, True),    # k = 32: four groups of eight loads
    (40, 5, 9, 3, 16, False),
    (1, 1, 4, 2, 8, True),        # one vector per row
    (3, 3, 10, 4, 65536, True),   # long rows, small batch
    (73, 2, 16, 8, 4096, False),  # 146 row chunks of 4 KB: small-batch combine (148 SMs)
    (74, 2, 16, 8, 4096, False),  # 148: streaming combine
    (147, 2, 16, 8, 2048, False),
    (148, 2, 16, 8, 2048, False),
]


@pytest.mark.parametrize("T,k,E,bs,H,renorm", COMBINE_CASES)
def test_combine_parity(T, k, E, bs, H, renorm):
    dev = require_gpu()
    g = torch.Generator().manual_seed(T * k + H)
    x = torch.randn((T, E), generator=g).to(torch.bfloat16)
    w_ref, ids_ref = oracle.topk_softmax(bf16_bits(x), k, renorm)
    ref = oracle.align_permute(ids_ref, E, bs)
    C = ref["capacity"]
    y = I.make_expert_out(C, H, seed=5)
    want = oracle.combine(bf16_bits(y), w_ref, ref["inv_perm"])
    out = tdt.moe_combine(y.to(dev), torch.from_numpy(w_ref).to(dev), torch.from_numpy(ref["inv_perm"]).to(dev))
    d = ulp_distance_bf16(bf16_bits(out), want)
    assert d.max() <= COMBINE_MAX_ULP, d.max()
    assert d.max() == 0, f"expected bit-exact combine (same fma order), max ulp {d.max()}"


@pytest.mark.parametrize("T", [64, 400])  # small-batch and streaming combine
def test_combine_remote_slots_and_partial_sums(T):
    """Expert-parallel partial sums: remote slots (-1) add nothing; a token with none gets +0."""
    dev = require_gpu()
    k, H = 6, 512
    rng = np.random.default_rng(1)
    C = 200
    inv = rng.integers(-1, C, size=T * k).astype(np.int32)
    inv[:k] = -1  # token 0 is all remote
    w = rng.uniform(0, 1, size=(T, k)).astype(np.float32)
    y = I.make_expert_out(C, H, seed=9)
    want = oracle.combine(bf16_bits(y), w, inv)
    out = tdt.moe_combine(y.to(dev), torch.from_numpy(w).to(dev), torch.from_numpy(inv).to(dev))
    got = bf16_bits(out)
    assert np.array_equal(got, want)
    assert (got[0] == 0).all()


@pytest.mark.parametrize("T", [8, 400])  # small-batch and streaming combine
def test_bad_rows_are_skipped_and_flagged(T):
    dev = require_gpu()
    k, H, C = 2, 64, 10
    base = [0, 1, 2, 99, 4, 5, -7, 7, 8, 9, 1, 2, 3, 4, 5, 6]
    inv = torch.tensor([base[i % 16] for i in range(T * k)], dtype=torch.int32)
    w = torch.full((T, k), 0.5)
    y = I.make_expert_out(C, H, seed=2)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    out = tdt.moe_combine(y.to(dev), w.to(dev), inv.to(dev), device_status=status)
    assert tdt.moe_read_status(status) == tdt.MOE_ERR_BAD_ROW
    ok = inv.clone()
    ok[(ok < -1) | (ok >= C)] = -1
    want = oracle.combine(bf16_bits(y), w.numpy(), ok.numpy())
    assert np.array_equal(bf16_bits(out), want)
    hidden = I.make_hidden(I.WORKLOADS["tiny_T64_E8_k2"], T=T, H=H)
    perm = torch.zeros((C, H), dtype=torch.bfloat16, device=dev)
    tdt.moe_gather(hidden.to(dev), k, inv.to(dev), C, permuted=perm, device_status=status)
    assert tdt.moe_read_status(status) == tdt.MOE_ERR_BAD_ROW
