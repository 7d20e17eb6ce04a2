"""Guard bands: every output of every entry point is written inside a larger buffer whose words before
and after the output hold a canary pattern; after the call the canaries must be intact (no write lands
outside an output) and the outputs must equal those of the same call on plain buffers.  Shapes cover
the single-kernel decode path, the tiled path with one warp per row and with lanes per row, ragged
tails, an expert map with remote slots, zero-filled pad rows and the expert-parallel reduce."""
import numpy as np
import pytest
import torch

import token_dispatch_topk_b200 as tdt
from token_dispatch_topk_b200 import binding as B

from gpu_helpers import require_gpu

pytestmark = pytest.mark.gpu

PAD_BYTES = 512
CANARY_I32 = -0x5A5A5A5B
CANARY_BF16_BITS = 0x7FA5  # a NaN pattern no kernel writes


class Guarded:
    """A tensor view with PAD_BYTES of canaries before and after it."""

    def __init__(self, shape, dtype, device):
        esz = torch.tensor([], dtype=dtype).element_size()
        pad = PAD_BYTES // esz
        n = int(np.prod(shape)) if len(shape) else 1
        self.big = torch.empty(pad + n + pad, dtype=dtype, device=device)
        if dtype == torch.bfloat16:
            self.big.view(torch.int16).fill_(CANARY_BF16_BITS)
        elif dtype == torch.float32:
            self.big.view(torch.int32).fill_(CANARY_I32)
        else:
            self.big.fill_(CANARY_I32)
        self.pad, self.n = pad, n
        self.view = self.big[pad:pad + n].view(*shape)

    def intact(self) -> bool:
        bf16 = self.big.dtype == torch.bfloat16
        w = self.big.view(torch.int16) if bf16 else self.big.view(torch.int32)
        want = CANARY_BF16_BITS if bf16 else CANARY_I32
        return bool((w[:self.pad] == want).all()) and bool((w[self.pad + self.n:] == want).all())


def _align_guarded(T, k, El, bs, dev):
    C = tdt.moe_align_capacity(T, k, El, bs)
    NB = tdt.moe_align_num_blocks(T, k, El, bs)
    g = [Guarded((El,), torch.int32, dev), Guarded((El + 1,), torch.int32, dev), Guarded((C,), torch.int32, dev),
         Guarded((NB,), torch.int32, dev), Guarded((1,), torch.int32, dev), Guarded((T * k,), torch.int32, dev)]
    return g, B.AlignResult(*(x.view for x in g), C)


CASES = [
    # name, T, E, k, dtype, E_local, map, bs, H
    ("decode_single_kernel", 2, 160, 6, torch.bfloat16, 40, "rank1", 8, 4096),
    ("tiled_warp_per_row_ragged", 333, 128, 8, torch.bfloat16, 128, None, 16, 264),
    ("tiled_lanes_fp32", 1500, 60, 4, torch.float32, 60, None, 64, 64),
    ("tiled_map_remote", 777, 64, 4, torch.bfloat16, 16, "rank1", 16, 128),
]


@pytest.mark.parametrize("name,T,E,k,dtype,El,mapkind,bs,H", CASES, ids=[c[0] for c in CASES])
def test_dispatch_and_stage_calls_stay_inside_their_outputs(name, T, E, k, dtype, El, mapkind, bs, H):
    dev = require_gpu()
    g = torch.Generator().manual_seed(T + E)
    x = torch.randn((T, E), generator=g).to(dtype).to(dev)
    hidden = torch.randn((T, H), generator=g).to(torch.bfloat16).to(dev)
    emap = None
    if mapkind == "rank1":
        m = torch.full((E,), -1, dtype=torch.int32)
        m[El:2 * El] = torch.arange(El, dtype=torch.int32)
        emap = m.to(dev)
    C = tdt.moe_align_capacity(T, k, El, bs)
    # the fused dispatch
    gw, gi = Guarded((T, k), torch.float32, dev), Guarded((T, k), torch.int32, dev)
    ga, al = _align_guarded(T, k, El, bs, dev)
    gp = Guarded((C, H), torch.bfloat16, dev)
    ws = tdt.alloc_dispatch_workspace(T, k, El, dev)
    tdt.moe_route_dispatch(x, hidden, k, True, bs, emap, El, topk_weights=gw.view, topk_ids=gi.view, align=al,
                           permuted=gp.view, workspace=ws)
    w_ref, ids_ref, al_ref, p_ref = tdt.moe_route_dispatch(x, hidden, k, True, bs, emap, El)
    torch.cuda.synchronize()
    for gg in [gw, gi, gp] + ga:
        assert gg.intact(), name
    assert torch.equal(gw.view, w_ref) and torch.equal(gi.view, ids_ref)
    for a, b in zip(al[:6], al_ref[:6]):
        assert torch.equal(a, b)
    npad = int(al_ref.num_tokens_post_pad.item())
    real = al_ref.sorted_token_ids[:npad] != T * k
    assert torch.equal(gp.view[:npad][real], p_ref[:npad][real])
    # the stage calls: gating, align, gather with zero-filled pads, combine
    gw2, gi2 = Guarded((T, k), torch.float32, dev), Guarded((T, k), torch.int32, dev)
    tdt.moe_topk_softmax(x, k, True, gw2.view, gi2.view)
    ga2, al2 = _align_guarded(T, k, El, bs, dev)
    tdt.moe_align_permute(gi2.view, E, bs, emap, El, out=al2)
    gp2 = Guarded((C, H), torch.bfloat16, dev)
    tdt.moe_gather(hidden, k, al2.inv_perm, C, sorted_token_ids=al2.sorted_token_ids,
                   num_tokens_post_pad=al2.num_tokens_post_pad, zero_pad=True, permuted=gp2.view)
    y = torch.randn((C, H), generator=g).to(torch.bfloat16).to(dev)
    go = Guarded((T, H), torch.bfloat16, dev)
    tdt.moe_combine(y, gw2.view, al2.inv_perm, out=go.view)
    out_ref = tdt.moe_combine(y, w_ref, al_ref.inv_perm)
    torch.cuda.synchronize()
    for gg in [gw2, gi2, gp2, go] + ga2:
        assert gg.intact(), name
    assert torch.equal(go.view, out_ref)
    pads = (al2.sorted_token_ids[:npad] == T * k)
    assert bool((gp2.view[:npad][pads].view(torch.int16) == 0).all())  # zero-filled pads, +0
    assert tdt.moe_read_status(ws) == tdt.MOE_OK


def test_reduce_partials_stays_inside_its_output():
    dev = require_gpu()
    g = torch.Generator().manual_seed(3)
    parts = [torch.randn((129, 72), generator=g).to(torch.bfloat16).to(dev) for _ in range(3)]
    go = Guarded((129, 72), torch.bfloat16, dev)
    tdt.moe_reduce_partials(parts, out=go.view)
    ref = tdt.moe_reduce_partials(parts)
    torch.cuda.synchronize()
    assert go.intact() and torch.equal(go.view, ref)
