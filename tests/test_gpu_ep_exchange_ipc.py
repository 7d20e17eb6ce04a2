"""The expert-parallel exchange through the owners' memory (dist.EpExchange), run as two and three
processes (ranks) on one GPU: the receive buffers are shared between the processes through CUDA IPC,
each rank's moe_combine writes its partial's token ranges into the owners' buffers, a process-group
barrier (gloo) orders those stores before the reads, and each owner runs moe_reduce_partials.

No kernel here waits for another process's kernel: the only cross-rank waits are on the host.  On
several GPUs the same code writes over NVLink; here it checks the buffer sharing, the slot layout,
the barrier placement and the alternating buffers.  Bars: each owner's rows equal the oracle's reduce
of the ranks' partials (bit-exact); each partial equals the oracle's combine of that rank's slots.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle

pytestmark = pytest.mark.gpu

E, K, H, BS, STEPS = 48, 6, 136, 8, 3


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _worker(rank, world, T, port, q):
    import torch.distributed as dist
    import token_dispatch_topk_b200 as tdt
    from token_dispatch_topk_b200 import dist as D
    from token_dispatch_topk_b200 import inputs as I
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        # the same routes on every rank: seeded logits, gated on the GPU
        logits = (I.normal_range(11, 0, T * E).view(T, E)).to(torch.bfloat16)
        w, ids = tdt.moe_topk_softmax(logits.to(dev), K, True)
        emap, El = D.ep_expert_map(E, world, rank)
        al = tdt.moe_align_permute(ids, E, BS, emap.to(dev), El)
        ex = D.EpExchange(T, H, dev)
        res = {"w": w.cpu().numpy(), "ids": ids.cpu().numpy(), "inv_perm": al.inv_perm.cpu().numpy(),
               "logits": _bits(logits), "outs": [], "ys": [], "partials": []}
        for step in range(STEPS):
            y = I.make_expert_out(al.capacity, H, seed=10 * step + rank, device=dev)  # this rank's expert outputs
            out = ex.combine_reduce(y, w, al.inv_perm)
            torch.cuda.synchronize()
            res["outs"].append(_bits(out))
            res["ys"].append(_bits(y))
            res["partials"].append(_bits(tdt.moe_combine(y, w, al.inv_perm)))
        q.put((rank, res))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("T,world", [(301, 2), (301, 3), (2, 3)], ids=["T301_two_ranks", "T301_three_ranks",
                                                                      "decode_T2_owner_without_tokens"])
def test_ep_exchange_through_ipc_on_one_gpu(T, world):
    assert torch.cuda.is_available()
    oracle.default()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, T, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    from token_dispatch_topk_b200 import dist as D
    w_ref, ids_ref = oracle.topk_softmax(res[0]["logits"], K, True)
    for r in range(world):
        assert np.array_equal(res[r]["ids"], ids_ref)
        emap, El = D.ep_expert_map(E, world, r)
        al = oracle.align_permute(ids_ref, E, BS, emap.numpy(), El)
        assert np.array_equal(res[r]["inv_perm"], al["inv_perm"])
    for step in range(STEPS):
        partials = []
        for r in range(world):
            want = oracle.combine(res[r]["ys"][step], res[r]["w"], res[r]["inv_perm"])
            assert np.array_equal(res[r]["partials"][step], want), (step, r)
            partials.append(want)
        full = oracle.reduce_partials(np.stack(partials))
        for o in range(world):
            lo, hi = D.ep_token_range(T, world, o)
            assert np.array_equal(res[o]["outs"][step], full[lo:hi]), (step, o)
