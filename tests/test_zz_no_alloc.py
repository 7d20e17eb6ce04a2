"""moe_align_permute_noalloc, the align entry point for callers that cannot allocate device memory
(their framework hands a custom op only its inputs and outputs, and no cudaMalloc is allowed while
it runs).  It keeps its scratch in a fixed per-GPU array inside the library instead of a caller
workspace.

Checked through the C ABI against moe_align_permute with a workspace and against the CPU oracle's
align, on the same inputs, for two calls in a row (the second call finds the previous call's
leftovers in the shared array).  The bar is the align bar: every output bit-exact.  The cases cover
no tokens, more than 512 local experts at mid sizes (where moe_align_permute runs other kernels)
and a size just under the array's limit.  This file is collected last; it passes on its own in a
fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

import oracle
import token_dispatch_topk_b200 as tdt
from token_dispatch_topk_b200 import binding as B
from token_dispatch_topk_b200 import inputs as I

pytestmark = pytest.mark.gpu

FIELDS = ("counts", "offsets", "sorted_token_ids", "expert_ids", "num_tokens_post_pad", "inv_perm")

CASES = [
    # name, T, k, E_global, map kind, E_local, block_size
    ("single_tile", 64, 2, 8, None, 8, 16),
    ("decode_rank_map", 2, 6, 160, "rank1", 40, 8),
    ("prefill_multi_tile", 4096, 8, 128, None, 128, 64),
    ("ragged_bad_ids", 5001, 3, 64, "rank1_bad", 16, 16),
    ("skewed_65536_tokens", 65536, 8, 256, "zipf", 256, 128),
    ("no_tokens", 0, 4, 32, None, 32, 16),
    ("many_local_experts_mid_size", 3000, 6, 900, "strided", 700, 32),
    ("thousand_experts_tile_path", 8192, 4, 1024, None, 1024, 64),
    # E_local = 1024 and 255 tiles of 8192 slots: 256 + 255 * 1024 * 4 bytes of scratch, just under 1 MiB
    ("just_under_scratch_limit", 522240, 4, 1024, None, 1024, 16),
]


def _inputs(kind, T, k, E, E_local, seed):
    g = np.random.default_rng(seed)
    emap = None
    if kind in ("rank1", "rank1_bad"):
        emap = np.full(E, -1, np.int32)
        emap[E_local:2 * E_local] = np.arange(E_local, dtype=np.int32)
    if kind == "strided":  # every other expert remote, 700 of 900 local
        emap = np.full(E, -1, np.int32)
        emap[np.arange(E_local) * E // E_local] = np.arange(E_local, dtype=np.int32)
    if kind == "zipf":
        wl = I.WORKLOADS["zipf_prefill_T65536_E256_k8_H7168"]
        logits = I.make_logits(wl).cuda()
        _, ids = tdt.moe_topk_softmax(logits, wl.k, wl.renormalize)
        return emap, ids
    lo, hi = (-2, E + 2) if kind == "rank1_bad" else (0, E)
    return emap, torch.from_numpy(g.integers(lo, hi, size=(T, k)).astype(np.int32)).cuda()


@pytest.mark.parametrize("name,T,k,E,kind,E_local,bs", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_workspace_entry_point(name, T, k, E, kind, E_local, bs):
    assert torch.cuda.is_available()
    emap, ids = _inputs(kind, T, k, E, E_local, seed=T + k)
    emap_d = None if emap is None else torch.from_numpy(emap).cuda()
    ref = tdt.moe_align_permute(ids, E, bs, emap_d, E_local)
    ref_status = tdt.moe_read_status(tdt.alloc_workspace(T, k, E_local, ids.device))  # a fresh word: 0
    assert ref_status == tdt.MOE_OK
    torch.cuda.synchronize()
    orc = oracle.align_permute(ids.cpu().numpy().reshape(T, k), E, bs, emap, E_local)
    for call in range(2):
        status = torch.zeros(1, dtype=torch.int32, device=ids.device)
        out = B.alloc_align_outputs(T, k, E_local, bs, ids.device)
        for f in FIELDS:  # poison the outputs so that every element must be written
            getattr(out, f).fill_(-12345)
        tdt.moe_align_permute_noalloc(ids, E, bs, emap_d, E_local, out=out, device_status=status)
        torch.cuda.synchronize()
        for f in FIELDS:
            assert torch.equal(getattr(out, f), getattr(ref, f)), f"{name}, call {call}: {f} differs"
            assert np.array_equal(getattr(out, f).cpu().numpy(), orc[f]), f"{name}, call {call}: {f} vs oracle"
        want = tdt.MOE_ERR_BAD_EXPERT_ID if kind == "rank1_bad" else tdt.MOE_OK
        assert tdt.moe_read_status(status) == want


def test_noalloc_rejects_sizes_beyond_its_scratch():
    assert torch.cuda.is_available()
    lib = B.load_library()
    T, k, E = 1 << 18, 4, 1024  # 1M slots, 1024 local experts: about 2 MiB of tile counters
    assert tdt.moe_align_workspace_bytes(T, k, E) > (1 << 20)
    buf = torch.empty(16, dtype=torch.int32, device="cuda")
    p = buf.data_ptr()
    st = lib.moe_align_permute_noalloc(p, T, k, E, None, E, 64, p, p, p, p, p, p, None, None)
    assert st == tdt.MOE_ERR_UNSUPPORTED
    # one token past the largest case above: 256 tiles of 8192 slots, 256 bytes over the array
    st = lib.moe_align_permute_noalloc(p, 522241, 4, E, None, E, 16, p, p, p, p, p, p, None, None)
    assert st == tdt.MOE_ERR_UNSUPPORTED
