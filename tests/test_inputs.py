"""The seeded input generators: deterministic, the documented shapes and distributions, and the
counter-based generator pinned to SplitMix64's published outputs and to the Irwin-Hall moments."""
import numpy as np
import pytest
import torch

from token_dispatch_topk_b200 import inputs as I

import oracle_pins


def test_workload_table():
    names = set(I.WORKLOADS)
    assert I.DEFAULT_WORKLOAD in names and len(names) == 5
    assert set(I.BENCH_SUB_WORKLOADS) | {I.DEFAULT_WORKLOAD, "tiny_T64_E8_k2"} == names
    wl = I.WORKLOADS[I.DEFAULT_WORKLOAD]  # the largest workload
    assert (wl.T, wl.E, wl.k, wl.H, wl.block_size, wl.renormalize) == (65536, 256, 8, 7168, 128, True)
    wl = I.WORKLOADS["qwen3moe_prefill_T4096_E128_k8"]
    assert (wl.T, wl.E, wl.k, wl.H, wl.block_size, wl.renormalize) == (4096, 128, 8, 2048, 64, True)
    dec = I.WORKLOADS["ep_decode_T2_E160_local40_k6"]
    m = I.expert_map(dec)
    assert m.tolist() == oracle_pins.rank1_of_4_map(160, 40, 1).tolist()


def test_deterministic_and_dtyped():
    wl = I.WORKLOADS["tiny_T64_E8_k2"]
    a, b = I.make_logits(wl), I.make_logits(wl)
    assert a.dtype == torch.bfloat16 and a.shape == (64, 8) and torch.equal(a, b)
    assert not torch.equal(I.make_logits(wl, seed=1), a)
    h = I.make_hidden(wl)
    assert h.shape == (64, 256) and torch.equal(h, I.make_hidden(wl))
    f = I.make_logits(I.WORKLOADS["nonpow2_T16384_E60_k4"], T=4096)
    assert f.dtype == torch.float32 and abs(float(f.var()) - 2.0) < 0.1  # N(0, 2): variance 2


def test_zipf_bias_is_skewed():
    wl = I.WORKLOADS["zipf_prefill_T65536_E256_k8_H7168"]
    b = I.zipf_bias(wl)
    assert b.shape == (256,) and float(b.max()) == 0.0
    ranks = np.sort(np.exp(-b.numpy().astype(np.float64) / 1.1))  # recover the ranks 1..E
    assert np.allclose(ranks, np.arange(1, 257), rtol=1e-5)
    x = I.make_logits(wl, T=2048).float()
    top = x.argmax(1)
    hot = int(b.argmax())
    assert (top == hot).float().mean() > 0.2  # the hottest expert wins far more than 1/256 of rows


def test_decode_patterns_match_golden():
    g = oracle_pins.load_golden("decode_route_patterns.json")
    assert set(g["patterns"]) == set(I.DECODE_PATTERNS)
    for name, pat in g["patterns"].items():
        assert I.decode_pattern_ids(name).tolist() == pat["ids"]


def test_strided_map():
    m = I.strided_expert_map(16, 4, 1)
    assert m.tolist() == [-1, 0, -1, -1, -1, 1, -1, -1, -1, 2, -1, -1, -1, 3, -1, -1]


def test_splitmix64_published_outputs():
    """SplitMix64 started at state 0 gives 0xe220a8397b1dcdaf, 0x6e789e6aa1b965f4, 0x06c45d188009454f
    (the reference generator's first three outputs); the tensor form agrees with the Python-int form."""
    G = 0x9E3779B97F4A7C15
    want = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    assert [I.mix64_int(n * G) for n in (1, 2, 3)] == want
    got = I._mix64_(torch.tensor([I._as_i64(n * G) for n in (1, 2, 3)], dtype=torch.int64))
    assert [int(v) & ((1 << 64) - 1) for v in got] == want
    rng = np.random.default_rng(4)
    vals = [int(v) for v in rng.integers(0, 1 << 63, 64, dtype=np.int64)] + [(1 << 64) - 1, 1 << 63, 0]
    got = I._mix64_(torch.tensor([I._as_i64(v) for v in vals], dtype=torch.int64))
    assert [int(v) & ((1 << 64) - 1) for v in got] == [I.mix64_int(v) for v in vals]


def test_stream_draws_are_the_splitmix_sequence_from_the_key():
    """Draw n of a stream is the (n+1)-th SplitMix64 output after the stream key."""
    for sid in (0, 1, 6, 123):
        state = I.stream_key(sid)
        seq = []
        for _ in range(5):
            state = (state + 0x9E3779B97F4A7C15) & ((1 << 64) - 1)
            seq.append(I.mix64_int(state))
        got = I.draws(sid, torch.arange(5, dtype=torch.int64))
        assert [int(v) & ((1 << 64) - 1) for v in got] == seq


def test_irwin_hall_values_and_moments():
    """z = (sum of twelve 16-bit fields - 393210) / 2^16: exact multiples of 2^-16 inside (-6, 6), with the
    moments of Irwin-Hall(12) - 6 (mean 0, variance 1, excess kurtosis -1/10)."""
    z = I.normal_range(5, 0, 1 << 21).double()
    assert torch.equal(z * 65536, torch.round(z * 65536)) and float(z.abs().max()) < 6
    m, v = float(z.mean()), float(z.var())
    assert abs(m) < 4e-3 and abs(v - 1) < 4e-3
    kurt = float(((z - m) ** 4).mean() / v ** 2) - 3
    assert abs(kurt + 0.1) < 0.02
    # element i from its own three draws, summed field by field
    i = 777
    d = [int(x) & ((1 << 64) - 1) for x in I.draws(5, torch.tensor([3 * i, 3 * i + 1, 3 * i + 2]))]
    s = sum((w >> sh) & 0xFFFF for w in d for sh in (0, 16, 32, 48))
    assert float(z[i]) == (s - 393210) / 65536


def test_rows_regenerate_by_index():
    wl = I.WORKLOADS["tiny_T64_E8_k2"]
    h = I.make_hidden(wl)
    toks = torch.tensor([63, 0, 17, 17])
    assert torch.equal(I.hidden_rows(toks, wl.H), h[toks])
    y = I.make_expert_out(100, 16)
    rows = torch.tensor([99, 3, 50])
    assert torch.equal(I.expert_out_rows(rows, 16), y[rows])
    assert torch.equal(I.make_hidden(wl, T=10), h[:10])
    assert not torch.equal(I.make_expert_out(100, 16, seed=1), y)


def test_decode_weights_are_uniform_draws():
    w = I.decode_pattern_weights()
    assert w.shape == (2, 6) and float(w.min()) >= 0 and float(w.max()) < 1
    assert torch.equal(w * 16777216, torch.round(w * 16777216))
