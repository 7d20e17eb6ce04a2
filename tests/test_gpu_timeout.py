"""Failure detection without a GPU fault: a bounded wait that runs out.

Every wait in the library's kernels has a time limit.  A test hook in the dispatch workspace
header (word 2: withhold bits, word 3: the limit in microseconds; both zero in normal use)
withholds the one event a wait depends on, so the wait runs out after a short limit.  The kernel
must then record MOE_ERR_TIMEOUT in the status word and return (no hang, no fault, no copies left
in flight), and the next call on the same workspace, with the hooks cleared, must be correct.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import token_dispatch_topk_b200 as tdt
from token_dispatch_topk_b200 import binding as B
from token_dispatch_topk_b200 import inputs as I

from gpu_helpers import assert_align_equal, bf16_bits, logits_for_oracle, np_i32, require_gpu

pytestmark = pytest.mark.gpu

HOOK_WITHHOLD_ROW_LOADS = 1  # placement + gather kernel: the hidden-row loads are never issued
LIMIT_US = 20000


def _check_step_against_oracle(r, wl, logits, hidden, what):
    w_ref, ids_ref = oracle.topk_softmax(logits_for_oracle(logits), wl.k, wl.renormalize)
    assert np.array_equal(np_i32(r.topk_ids), ids_ref), what
    al = oracle.align_permute(ids_ref, wl.E, wl.block_size)
    assert_align_equal(r.align, al, what)
    npad = int(al["num_tokens_post_pad"][0])
    perm = oracle.gather(bf16_bits(hidden), wl.k, al["sorted_token_ids"], npad, al["capacity"])
    real = al["sorted_token_ids"][:npad] != wl.T * wl.k
    assert np.array_equal(bf16_bits(r.permuted[:npad])[real], perm[:npad][real]), what


@pytest.mark.parametrize("name", ["tiny_T64_E8_k2", "qwen3moe_prefill_T4096_E128_k8"])
def test_withheld_row_loads_time_out_and_the_workspace_recovers(name):
    dev = require_gpu()
    wl = I.WORKLOADS[name]
    logits, hidden = I.make_logits(wl), I.make_hidden(wl)
    r = tdt.MoeRouter(wl.T, wl.E, wl.k, wl.H, wl.block_size, wl.renormalize, device=dev)
    assert not r.small_batch
    ws = r.dispatch_workspace
    ws[2] = HOOK_WITHHOLD_ROW_LOADS
    ws[3] = LIMIT_US
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    r.dispatch(logits.to(dev), hidden.to(dev))
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert B.moe_read_status(ws) == tdt.MOE_ERR_TIMEOUT
    assert elapsed < 1.0, f"the wait ran for {elapsed:.3f} s; its limit was {LIMIT_US} us"
    ws[2] = 0
    ws[3] = 0
    for f in ("sorted_token_ids", "inv_perm", "expert_ids", "counts", "offsets"):
        getattr(r.align, f).fill_(-7)
    r.dispatch(logits.to(dev), hidden.to(dev))
    torch.cuda.synchronize()
    assert B.moe_read_status(ws) == tdt.MOE_OK
    _check_step_against_oracle(r, wl, logits, hidden, f"{name} after the timeout")
