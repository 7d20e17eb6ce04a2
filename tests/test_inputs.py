"""The seeded input generators: deterministic, the documented shapes and distributions."""
import numpy as np
import pytest
import torch

from token_dispatch_topk_b200 import inputs as I

import oracle_pins


def test_workload_table():
    names = set(I.WORKLOADS)
    assert I.DEFAULT_WORKLOAD in names and len(names) == 5
    wl = I.WORKLOADS[I.DEFAULT_WORKLOAD]
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
    ranks = np.sort(np.exp(-b.numpy() / 1.1))  # recover the ranks 1..E
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


def test_expert_out_chunks_on_cpu():
    y = I.make_expert_out(100, 16, chunk_rows=32)
    assert y.shape == (100, 16) and y.dtype == torch.bfloat16
    assert torch.equal(y, I.make_expert_out(100, 16, chunk_rows=32))
