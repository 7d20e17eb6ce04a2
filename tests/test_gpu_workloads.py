"""End-to-end GPU parity on the five routing workloads, at their full sizes, through
MoeRouter.step (the four C-ABI calls the bench times) against the CPU oracle pipeline.

Every workload is compared in full.  The skewed 65 536-token workload (about 17 GB on the
device) is compared in chunks: every gathered row below N_pad against the oracle's gather of
that chunk's slot ids, and every combined token against the oracle's combine of that chunk of
tokens, the expert-output rows they read being copied back from the device.  The large inputs
are generated on the device by the counter-based generator (the same bits as on the host, which
tests/test_gpu_inputs.py checks) and copied back for the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import token_dispatch_topk_b200 as tdt
from token_dispatch_topk_b200 import inputs as I

from gpu_helpers import (COMBINE_MAX_ULP, TOPK_WEIGHT_ATOL, assert_align_equal,
                         assert_combine_within_weight_tolerance, bf16_bits, logits_for_oracle, np_i32, require_gpu,
                         ulp_distance_bf16)

pytestmark = pytest.mark.gpu

FULL = ["tiny_T64_E8_k2", "qwen3moe_prefill_T4096_E128_k8", "nonpow2_T16384_E60_k4"]


def _router(wl, dev):
    emap = I.expert_map(wl)
    return tdt.MoeRouter(wl.T, wl.E, wl.k, wl.H, wl.block_size, wl.renormalize, E_local=wl.E_local,
                         expert_map=emap, logits_dtype=torch.bfloat16 if wl.logits_dtype == "bf16" else torch.float32,
                         device=dev)


def _oracle_pipeline(wl, logits, hidden_bits, y_bits, ids_override=None, w_override=None):
    w, ids = oracle.topk_softmax(logits_for_oracle(logits), wl.k, wl.renormalize)
    if ids_override is not None:
        ids = ids_override
    if w_override is not None:
        w = w_override
    emap = I.expert_map(wl)
    al = oracle.align_permute(ids, wl.E, wl.block_size, None if emap is None else emap.numpy(), wl.experts_local)
    npad = int(al["num_tokens_post_pad"][0])
    perm = oracle.gather(hidden_bits, wl.k, al["sorted_token_ids"], npad, al["capacity"])
    out = oracle.combine(y_bits, w, al["inv_perm"])
    return w, ids, al, perm, out


def _check_all(r, wl, ref, what, y, y_bits):
    """Every stage of one GPU step against the oracle pipeline.

    The step's combine used the GPU gating weights: it is checked against the propagated weight
    tolerance, then re-run on the oracle's weights and required to match within 1 bf16 ulp."""
    w_ref, ids_ref, al_ref, perm_ref, out_ref = ref
    assert np.array_equal(np_i32(r.topk_ids), ids_ref), what
    assert np.abs(r.topk_weights.cpu().numpy() - w_ref).max() <= TOPK_WEIGHT_ATOL, what
    assert_align_equal(r.align, al_ref, what)
    npad = int(al_ref["num_tokens_post_pad"][0])
    real = al_ref["sorted_token_ids"][:npad] != wl.T * wl.k
    got = bf16_bits(r.permuted[:npad])
    assert np.array_equal(got[real], perm_ref[:npad][real]), what
    assert_combine_within_weight_tolerance(bf16_bits(r.out), out_ref, y_bits, al_ref["inv_perm"], wl.k, what)
    out2 = tdt.moe_combine(y, torch.from_numpy(w_ref).to(y.device), r.align.inv_perm)
    d = ulp_distance_bf16(bf16_bits(out2), out_ref)
    assert d.max() <= COMBINE_MAX_ULP, (what, d.max())


def _run(r, path, logits, hidden, y):
    return r.step_fused(logits, hidden, y) if path == "fused" else r.step_staged(logits, hidden, y)


@pytest.mark.parametrize("path", ["fused", "staged"])
@pytest.mark.parametrize("name", FULL)
def test_workload_full_size(name, path):
    dev = require_gpu()
    wl = I.WORKLOADS[name]
    logits = I.make_logits(wl)
    hidden = I.make_hidden(wl, device=dev).cpu()
    yd = I.make_expert_out(wl.capacity, wl.H, device=dev)
    y = yd.cpu()
    r = _router(wl, dev)
    _run(r, path, logits.to(dev), hidden.to(dev), yd)
    torch.cuda.synchronize()
    ref = _oracle_pipeline(wl, logits, bf16_bits(hidden), bf16_bits(y))
    _check_all(r, wl, ref, name, yd, bf16_bits(y))
    assert r.device_status() == tdt.MOE_OK


@pytest.mark.parametrize("path", ["fused", "staged"])
def test_ep_decode_every_route_pattern(path):
    """M=2, top-k 6, rank 1 of 4 (40 local experts): the logits-derived routing and every
    injected route pattern, including the valid all-remote rank."""
    dev = require_gpu()
    wl = I.WORKLOADS["ep_decode_T2_E160_local40_k6"]
    logits = I.make_logits(wl)
    hidden = I.make_hidden(wl)
    y = I.make_expert_out(wl.capacity, wl.H)
    r = _router(wl, dev)
    yd = y.to(dev)
    _run(r, path, logits.to(dev), hidden.to(dev), yd)
    torch.cuda.synchronize()
    _check_all(r, wl, _oracle_pipeline(wl, logits, bf16_bits(hidden), bf16_bits(y)), "logits-derived", yd,
               bf16_bits(y))
    w_inj = I.decode_pattern_weights()
    for name in I.DECODE_PATTERNS:
        ids = I.decode_pattern_ids(name)
        if path == "fused":
            r.step_routes(ids.to(dev), w_inj.to(dev), hidden.to(dev), y.to(dev))
        else:
            r.gate(logits.to(dev))
            r.topk_ids.copy_(ids.to(dev))
            r.topk_weights.copy_(w_inj.to(dev))
            r.align_permute()
            r.gather(hidden.to(dev))
            r.combine(y.to(dev))
        torch.cuda.synchronize()
        w_ref, _, al, perm, out = _oracle_pipeline(wl, logits, bf16_bits(hidden), bf16_bits(y),
                                                   ids_override=ids.numpy(), w_override=w_inj.numpy())
        assert_align_equal(r.align, al, name)
        npad = int(al["num_tokens_post_pad"][0])
        real = al["sorted_token_ids"][:npad] != wl.T * wl.k
        assert np.array_equal(bf16_bits(r.permuted[:npad])[real], perm[:npad][real]), name
        assert np.array_equal(bf16_bits(r.out), out), name
        if name == "all_remote":
            assert npad == 0 and (bf16_bits(r.out) == 0).all()


@pytest.mark.parametrize("path", ["fused", "staged"])
def test_skewed_prefill_full_size(path):
    dev = require_gpu()
    wl = I.WORKLOADS["zipf_prefill_T65536_E256_k8_H7168"]
    T, k, H = wl.T, wl.k, wl.H
    logits = I.make_logits(wl)
    hidden_d = I.make_hidden(wl, device=dev)
    y_dev = I.make_expert_out(wl.capacity, wl.H, device=dev)
    r = _router(wl, dev)
    _run(r, path, logits.to(dev), hidden_d, y_dev)
    torch.cuda.synchronize()
    assert r.device_status() == tdt.MOE_OK
    # gating and align in full
    w_ref, ids_ref = oracle.topk_softmax(logits_for_oracle(logits), k, wl.renormalize)
    assert np.array_equal(np_i32(r.topk_ids), ids_ref)
    assert np.abs(r.topk_weights.cpu().numpy() - w_ref).max() <= TOPK_WEIGHT_ATOL
    al = oracle.align_permute(ids_ref, wl.E, wl.block_size)
    assert_align_equal(r.align, al, "skewed")
    counts = al["counts"]
    assert counts.max() > 8 * counts.mean()  # the Zipf bias makes a few experts hot
    # gather: every row below N_pad, chunk by chunk, against the oracle's gather of the chunk's slot ids
    hidden_bits = bf16_bits(hidden_d)
    npad = int(al["num_tokens_post_pad"][0])
    rows_per_chunk = 1 << 15
    for p0 in range(0, npad, rows_per_chunk):
        p1 = min(npad, p0 + rows_per_chunk)
        sti = al["sorted_token_ids"][p0:p1]
        want = oracle.gather(hidden_bits, k, sti, p1 - p0, p1 - p0)
        got = bf16_bits(r.permuted[p0:p1])
        real = sti != T * k
        assert np.array_equal(got[real], want[real]), f"gathered rows {p0}..{p1}"
    del hidden_bits
    # combine: every token, chunk by chunk; the expert-output rows a chunk reads are copied back
    out2 = tdt.moe_combine(y_dev, torch.from_numpy(w_ref).to(dev), r.align.inv_perm)
    torch.cuda.synchronize()
    inv = al["inv_perm"].reshape(T, k)
    toks_per_chunk = 2048
    for t0 in range(0, T, toks_per_chunk):
        t1 = min(T, t0 + toks_per_chunk)
        inv_c = inv[t0:t1]
        used = np.unique(inv_c[inv_c >= 0])
        y_rows = bf16_bits(y_dev[torch.from_numpy(used).long().to(dev)])
        remap = np.full(wl.capacity, -1, np.int64)
        remap[used] = np.arange(len(used))
        inv_r = np.where(inv_c >= 0, remap[np.maximum(inv_c, 0)], -1).astype(np.int32).reshape(-1)
        want = oracle.combine(y_rows, w_ref[t0:t1], inv_r)
        # the step's combine used the GPU gating weights: the propagated weight tolerance
        assert_combine_within_weight_tolerance(bf16_bits(r.out[t0:t1]), want, y_rows, inv_r, k,
                                               f"skewed tokens {t0}..{t1}")
        # the combine on the oracle's weights: within 1 bf16 ulp
        d = ulp_distance_bf16(bf16_bits(out2[t0:t1]), want)
        assert d.max() <= COMBINE_MAX_ULP, (t0, d.max())


@pytest.mark.parametrize("name", ["qwen3moe_prefill_T4096_E128_k8", "ep_decode_T2_E160_local40_k6"])
def test_repeat_steps_are_bit_identical(name):
    """Repeated steps, alternating the staged and the fused dispatch, give the same bits."""
    dev = require_gpu()
    wl = I.WORKLOADS[name]
    logits, hidden = I.make_logits(wl, device=dev), I.make_hidden(wl, device=dev)
    y = I.make_expert_out(wl.capacity, wl.H, device=dev)
    r = _router(wl, dev)
    first = None
    for i in range(6):
        (r.step_staged if i % 2 == 0 else r.step_fused)(logits, hidden, y)
        snap = [t.clone() for t in (r.topk_ids, r.topk_weights, r.align.sorted_token_ids, r.align.inv_perm,
                                    r.align.expert_ids, r.out)]
        if first is None:
            first = snap
        else:
            for a, b in zip(first, snap):
                assert torch.equal(a, b)


def test_end_to_end_from_host_buffers():
    dev = require_gpu()
    wl = I.WORKLOADS["tiny_T64_E8_k2"]
    logits, hidden = I.make_logits(wl).pin_memory(), I.make_hidden(wl).pin_memory()
    y = I.make_expert_out(wl.capacity, wl.H)
    out_host = torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory()
    r = _router(wl, dev)
    r.step_from_host(logits, hidden, y.to(dev), out_host)
    torch.cuda.synchronize()
    ref = _oracle_pipeline(wl, logits, bf16_bits(hidden), bf16_bits(y))
    assert np.array_equal(np_i32(r.topk_ids), ref[1])
    assert_combine_within_weight_tolerance(bf16_bits(out_host), ref[4], bf16_bits(y), ref[2]["inv_perm"], wl.k,
                                           "from host")


def test_zero_tokens():
    dev = require_gpu()
    r = tdt.MoeRouter(0, 16, 4, 64, 8, True, device=dev)
    r.step(torch.empty((0, 16), dtype=torch.bfloat16, device=dev), torch.empty((0, 64), dtype=torch.bfloat16,
                                                                                 device=dev),
           torch.empty((r.capacity, 64), dtype=torch.bfloat16, device=dev))
    torch.cuda.synchronize()
    ref = oracle.align_permute(np.zeros((0, 4), np.int32), 16, 8)
    assert_align_equal(r.align, ref, "T=0")


@pytest.mark.parametrize("name", ["tiny_T64_E8_k2", "qwen3moe_prefill_T4096_E128_k8"])
def test_host_step_pipeline_matches_serial_steps(name):
    """The double-buffered end-to-end path: five steps with different inputs in flight together give, for
    each step, the bits of the same step run alone, and step 0 matches the oracle."""
    dev = require_gpu()
    wl = I.WORKLOADS[name]
    y = I.make_expert_out(wl.capacity, wl.H, device=dev)
    ins = [(I.make_logits(wl, seed=s).pin_memory(), I.make_hidden(wl, seed=s).pin_memory()) for s in range(5)]
    outs = [torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory() for _ in range(5)]
    r = _router(wl, dev)
    pipe = tdt.HostStepPipeline(r, expert_out=y)
    for (lg, hd), o in zip(ins, outs):
        pipe.submit(lg, hd, o)
    pipe.synchronize()
    assert r.device_status() == tdt.MOE_OK
    solo = _router(wl, dev)
    for (lg, hd), o in zip(ins, outs):
        want = solo.step(lg.to(dev), hd.to(dev), y)
        torch.cuda.synchronize()
        assert torch.equal(o, want.cpu())
    lg, hd = ins[0]
    ref = _oracle_pipeline(wl, lg, bf16_bits(hd), bf16_bits(y))
    assert_combine_within_weight_tolerance(bf16_bits(outs[0]), ref[4], bf16_bits(y), ref[2]["inv_perm"], wl.k,
                                           "pipelined step 0")
