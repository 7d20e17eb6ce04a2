"""The counter-based input generator gives the same bits on the device as on the host, so inputs
generated on the GPU (the large hidden and expert-output buffers) can be handed to the CPU oracle.
Torch's integer operations, exact fp32 scaling and round-to-nearest-even bf16 conversion are the only
arithmetic involved; these checks make that identity a tested fact rather than an assumption."""
import pytest
import torch

from token_dispatch_topk_b200 import inputs as I

from gpu_helpers import require_gpu

pytestmark = pytest.mark.gpu


def test_draws_and_normals_match_host():
    dev = require_gpu()
    idx = torch.cat([torch.arange(0, 4096), torch.randint(0, 1 << 40, (4096,), generator=torch.Generator().manual_seed(3))])
    for sid in (0, 1, 2, 3, 9):
        assert torch.equal(I.draws(sid, idx.to(dev)).cpu(), I.draws(sid, idx))
        assert torch.equal(I.normal_at(sid, idx.to(dev)).cpu(), I.normal_at(sid, idx))
        assert torch.equal(I.uniform_at(sid, idx.to(dev)).cpu(), I.uniform_at(sid, idx))


@pytest.mark.parametrize("name", list(I.WORKLOADS))
def test_workload_inputs_match_host(name):
    dev = require_gpu()
    wl = I.WORKLOADS[name]
    T = min(wl.T, 512)
    assert torch.equal(I.make_logits(wl, T=T, device=dev).cpu(), I.make_logits(wl, T=T))
    assert torch.equal(I.make_hidden(wl, T=T, device=dev).cpu(), I.make_hidden(wl, T=T))
    # rows scattered over the full expert-output buffer, regenerated on the host one by one
    rows = torch.unique(torch.cat([torch.tensor([0, wl.capacity - 1]),
                                   torch.randint(0, wl.capacity, (64,), generator=torch.Generator().manual_seed(1))]))
    assert torch.equal(I.expert_out_rows(rows, wl.H, device=dev).cpu(), I.expert_out_rows(rows, wl.H))


def test_full_expert_out_buffer_rows_match_host():
    """The skewed workload's 8 GB expert-output buffer, generated on the device in chunks: sampled rows
    equal the host's regeneration of the same rows."""
    dev = require_gpu()
    wl = I.WORKLOADS["zipf_prefill_T65536_E256_k8_H7168"]
    y = I.make_expert_out(wl.capacity, wl.H, device=dev)
    rows = torch.unique(torch.cat([torch.tensor([0, 1, wl.capacity - 1]),
                                   torch.randint(0, wl.capacity, (32,), generator=torch.Generator().manual_seed(2))]))
    assert torch.equal(y[rows.to(dev)].cpu(), I.expert_out_rows(rows, wl.H))
    h = I.make_hidden(wl, device=dev)
    toks = torch.tensor([0, 12345, wl.T - 1])
    assert torch.equal(h[toks.to(dev)].cpu(), I.hidden_rows(toks, wl.H))
