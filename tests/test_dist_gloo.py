"""The multi-process path on the CPU: two gloo ranks (world size 2), no GPU.

  * data parallel: each rank gets its own seed, and the timing reduction returns the maximum
    over the ranks;
  * expert parallel: each rank owns a contiguous block of experts (``ep_expert_map``), routes the
    same tokens with its map (the oracle stands in for the rank's kernels here), combines its
    local slots into a bf16 partial, and ``ep_reduce_partials`` all-gathers the partials and sums
    them in rank order (the oracle's reduce stands in for moe_reduce_partials).
    The result must match the oracle's single-rank combine of all slots within the rounding of
    the two partials and the final sum; the expert outputs are a function of (global expert,
    token) so that every rank builds its own expert-grouped rows consistently.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from token_dispatch_topk_b200 import dist as D
from token_dispatch_topk_b200 import inputs as I

from oracle_pins import bf16_bits_to_f32, f32_to_bf16_bits


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _expert_rows(ids_rows_experts, tokens, H):
    """Expert output row of (global expert e, token t): bf16 values from a fixed formula."""
    e = np.asarray(ids_rows_experts, np.float64)[:, None]
    t = np.asarray(tokens, np.float64)[:, None]
    h = np.arange(H, dtype=np.float64)[None, :]
    v = np.sin(0.37 * e + 0.11 * h) * np.cos(0.23 * t - 0.05 * h) * 3.0
    return f32_to_bf16_bits(v.astype(np.float32))


def _rank_partial(logits_bits, T, E, k, H, bs, world, rank):
    """One expert-parallel rank: route with its map, build its expert-grouped rows, combine its slots."""
    w, ids = oracle.topk_softmax(logits_bits, k, True)
    emap, El = D.ep_expert_map(E, world, rank)
    al = oracle.align_permute(ids, E, bs, emap.numpy(), El)
    C = al["capacity"]
    inv = al["inv_perm"]
    y = np.zeros((C, H), np.uint16)
    rows = np.nonzero(inv >= 0)[0]
    if rows.size:
        y[inv[rows]] = _expert_rows(ids.reshape(-1)[rows], rows // k, H)
    return w, ids, oracle.combine(y, w, inv)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out = {"seed": D.rank_seed(5, rank), "max": D.max_over_ranks(1.5 + rank)}
        wl = I.WORKLOADS["tiny_T64_E8_k2"]
        T, E, k, H, bs = 24, 16, 4, 64, 8
        logits = I.make_logits(wl, T=T)  # bf16 [T, 8]: widen to 16 experts deterministically
        logits = torch.cat([logits, logits.flip(1) * 0.5], dim=1).contiguous()
        bits = logits.view(torch.int16).numpy().view(np.uint16)
        _, _, partial = _rank_partial(bits, T, E, k, H, bs, world, rank)
        def oracle_reduce(parts):  # the oracle stands in for moe_reduce_partials on the CPU
            bits = np.stack([p.view(torch.int16).numpy().view(np.uint16) for p in parts])
            return torch.from_numpy(oracle.reduce_partials(bits).view(np.int16)).view(torch.bfloat16)

        summed = D.ep_reduce_partials(torch.from_numpy(partial.view(np.int16)).view(torch.bfloat16),
                                      reduce=oracle_reduce)
        out["partial"] = partial
        out["summed"] = summed.view(torch.int16).numpy().view(np.uint16)
        out["bits"] = bits
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_ranks():
    oracle.default()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def test_data_parallel_seeds_and_max_over_ranks(two_ranks):
    assert two_ranks[0]["seed"] != two_ranks[1]["seed"]
    assert two_ranks[0]["max"] == two_ranks[1]["max"] == 2.5


def test_expert_parallel_partials_sum_to_the_full_combine(two_ranks):
    T, E, k, H, bs = 24, 16, 4, 64, 8
    bits = two_ranks[0]["bits"]
    assert np.array_equal(bits, two_ranks[1]["bits"])
    s0, s1 = two_ranks[0]["summed"], two_ranks[1]["summed"]
    assert np.array_equal(s0, s1), "every rank holds the same reduced output"
    # the all-gather baseline sums in rank order: bit-identical to the oracle's reduce of the partials
    both = np.stack([two_ranks[0]["partial"], two_ranks[1]["partial"]])
    assert np.array_equal(s0, oracle.reduce_partials(both))
    # single rank owning every expert
    w, ids, full = _rank_partial(bits, T, E, k, H, bs, 1, 0)
    p0 = bf16_bits_to_f32(two_ranks[0]["partial"]).astype(np.float64)
    p1 = bf16_bits_to_f32(two_ranks[1]["partial"]).astype(np.float64)
    got = bf16_bits_to_f32(s0).astype(np.float64)
    want = bf16_bits_to_f32(full).astype(np.float64)

    def ulp(x):  # one bf16 ulp at |x| (normal range)
        e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -120)))
        return 2.0 ** (e - 7)

    # each partial and the final sum are rounded once to bf16, the full combine once
    bound = 0.5 * (ulp(p0) + ulp(p1) + ulp(got) + ulp(want)) + 1e-6 * (np.abs(p0) + np.abs(p1))
    assert (np.abs(got - want) <= bound).all(), np.max(np.abs(got - want) - bound)
    # and the partials cover disjoint expert blocks: each slot is local on exactly one rank
    lo0, hi0 = D.ep_expert_range(E, 2, 0)
    lo1, hi1 = D.ep_expert_range(E, 2, 1)
    assert (lo0, hi0, lo1, hi1) == (0, 8, 8, 16)


def test_ep_expert_range_splits_evenly():
    assert [D.ep_expert_range(10, 4, r) for r in range(4)] == [(0, 3), (3, 6), (6, 8), (8, 10)]
    m, El = D.ep_expert_map(160, 4, 1)
    assert El == 40 and m[40].item() == 0 and m[79].item() == 39 and m[39].item() == -1 and m[80].item() == -1
    with pytest.raises(ValueError):
        D.ep_expert_range(3, 4, 0)


def test_ep_token_range_partitions_the_tokens():
    """The owners' token ranges of the reduce-scatter form cover [0, T) in order, without overlap,
    sizes differing by at most one (owners past T get empty ranges)."""
    for T in (0, 1, 2, 3, 7, 64, 4097):
        for world in (1, 2, 3, 4, 8):
            ranges = [D.ep_token_range(T, world, o) for o in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == T
            for (lo, hi), (lo2, _) in zip(ranges, ranges[1:]):
                assert hi == lo2
            sizes = [hi - lo for lo, hi in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0
    with pytest.raises(ValueError):
        D.ep_token_range(10, 4, 4)
    with pytest.raises(ValueError):
        D.ep_token_range(-1, 2, 0)


def test_reduce_scatter_of_the_oracle_partials_is_the_reduce():
    """The reduce-scatter form gives each owner the rows of the full reduce: reducing each owner's
    token range of the partials and concatenating equals reducing the whole partials (per element
    the same sum in the same rank order)."""
    rng = np.random.default_rng(5)
    world, T, H = 4, 11, 16
    parts = f32_to_bf16_bits(rng.standard_normal((world, T, H)).astype(np.float32))
    full = oracle.reduce_partials(parts)
    pieces = []
    for o in range(world):
        lo, hi = D.ep_token_range(T, world, o)
        pieces.append(oracle.reduce_partials(parts[:, lo:hi]) if hi > lo else np.zeros((0, H), np.uint16))
    assert np.array_equal(np.concatenate(pieces), full)


def test_combine_to_owners_slices_each_owner_range(monkeypatch):
    """Host logic of the reduce-scatter form on the CPU: ep_combine_to_owners hands moe_combine each
    owner's token range (weights, slot rows and destination); the oracle's combine stands in for the
    kernel here, so each owner's slot must hold exactly that range of the rank's partial, owners
    without tokens included."""
    from token_dispatch_topk_b200 import binding as B

    def oracle_combine(expert_out, topk_weights, inv_perm, out=None, device_status=None, stream=None):
        bits = expert_out.contiguous().view(torch.int16).numpy().view(np.uint16)
        res = oracle.combine(bits, topk_weights.numpy(), inv_perm.numpy())
        out.copy_(torch.from_numpy(res.view(np.int16)).view(torch.bfloat16))
        return out

    monkeypatch.setattr(B, "moe_combine", oracle_combine)
    rng = np.random.default_rng(3)
    for T, E, k, H, bs, world in [(50, 32, 4, 16, 4, 4), (2, 160, 6, 8, 8, 4), (7, 12, 2, 8, 2, 3)]:
        w, ids = oracle.topk_softmax(rng.standard_normal((T, E)).astype(np.float32), k, True)
        ranges = [D.ep_token_range(T, world, o) for o in range(world)]
        for r in range(world):
            m, El = D.ep_expert_map(E, world, r)
            al = oracle.align_permute(ids, E, bs, m.numpy(), El)
            y = f32_to_bf16_bits(rng.standard_normal((al["capacity"], H)).astype(np.float32))
            dests = [torch.full((hi - lo, H), 7.0, dtype=torch.bfloat16) for lo, hi in ranges]
            D.ep_combine_to_owners(torch.from_numpy(y.view(np.int16)).view(torch.bfloat16), torch.from_numpy(w),
                                   torch.from_numpy(al["inv_perm"]), dests)
            full = oracle.combine(y, w, al["inv_perm"])
            for (lo, hi), d in zip(ranges, dests):
                assert np.array_equal(d.view(torch.int16).numpy().view(np.uint16), full[lo:hi]), (T, r, lo)
