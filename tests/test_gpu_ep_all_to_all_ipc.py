"""The all-to-all form of the expert-parallel layer (dist.EpAllToAll), run as two and three processes
(ranks) on one GPU with buffers shared through CUDA IPC: every rank gates its own tokens; every owner
aligns all ranks' routes on its experts, pulls the hidden rows it needs from each rank, and writes its
partial combine of each rank's slots into that rank's receive buffer; each rank reduces its partials.

No kernel waits for another process's kernel: the cross-rank waits are host barriers.  Ranks hold
different token counts (one holds none).  Bars: routes and gathered rows bit-exact, weights within 2e-6,
every align output bit-exact, and each rank's output equal to the oracle's rank-ordered reduce of the
oracle's partial combines of the same expert outputs (bit-exact).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle

pytestmark = pytest.mark.gpu

E, K, H, BS, STEPS = 40, 4, 72, 4, 2
FIELDS = ("counts", "offsets", "sorted_token_ids", "expert_ids", "num_tokens_post_pad", "inv_perm")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _worker(rank, T_per_rank, port, q):
    import torch.distributed as dist
    from token_dispatch_topk_b200 import dist as D
    from token_dispatch_topk_b200 import inputs as I
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    world = len(T_per_rank)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        Tr = T_per_rank[rank]
        ex = D.EpAllToAll(T_per_rank, E, K, H, BS, True, dev)
        steps = []
        for step in range(STEPS):
            logits = I.normal_range(100 + 10 * step + rank, 0, Tr * E).view(Tr, E).to(torch.bfloat16)
            hidden = I.normal_range(200 + 10 * step + rank, 0, Tr * H).view(Tr, H).to(torch.bfloat16)
            ex.hidden[:Tr].copy_(hidden.to(dev))
            y = I.make_expert_out(ex.capacity, H, seed=16 * step + rank, device=dev)  # this owner's experts
            out = ex.step(logits.to(dev), y)
            torch.cuda.synchronize()
            steps.append({"logits": _bits(logits), "hidden": _bits(hidden), "y": _bits(y), "out": _bits(out),
                          "ids": ex.topk_ids[:Tr].cpu().numpy(), "w": ex.topk_weights[:Tr].cpu().numpy(),
                          "permuted": _bits(ex.permuted),
                          **{f: getattr(ex.align, f).cpu().numpy() for f in FIELDS}})
        q.put((rank, steps))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("T_per_rank", [[100, 57], [37, 64, 0]], ids=["two_ranks", "three_ranks_one_empty"])
def test_ep_all_to_all_through_ipc_on_one_gpu(T_per_rank):
    assert torch.cuda.is_available()
    oracle.default()
    from token_dispatch_topk_b200 import dist as D
    world = len(T_per_rank)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, T_per_rank, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    T_total = sum(T_per_rank)
    for step in range(STEPS):
        st = [res[r][step] for r in range(world)]
        for r in range(world):  # gating of each rank's own tokens
            w_ref, ids_ref = oracle.topk_softmax(st[r]["logits"].reshape(T_per_rank[r], E), K, True)
            assert np.array_equal(st[r]["ids"], ids_ref), (step, r)
            if T_per_rank[r]:
                assert np.abs(st[r]["w"] - w_ref).max() <= 2e-6, (step, r)
        ids_all = np.concatenate([st[r]["ids"] for r in range(world)]).reshape(T_total, K)
        hidden_all = np.concatenate([st[r]["hidden"].reshape(T_per_rank[r], H) for r in range(world)])
        off = np.cumsum([0] + T_per_rank)
        partials = [[None] * world for _ in range(world)]  # [rank][owner]
        for d in range(world):  # each owner: align of every rank's routes, gathered rows, partial combines
            emap, El = D.ep_expert_map(E, world, d)
            al = oracle.align_permute(ids_all, E, BS, emap.numpy(), El)
            for f in FIELDS:
                assert np.array_equal(st[d][f], al[f]), (step, d, f)
            npad = int(al["num_tokens_post_pad"][0])
            perm = oracle.gather(hidden_all, K, al["sorted_token_ids"], npad, al["capacity"])
            real = al["sorted_token_ids"][:npad] != T_total * K
            assert np.array_equal(st[d]["permuted"][:npad][real], perm[:npad][real]), (step, d)
            y = st[d]["y"]
            for r in range(world):
                inv = al["inv_perm"][off[r] * K:off[r + 1] * K]
                partials[r][d] = oracle.combine(y, st[r]["w"].reshape(T_per_rank[r], K), inv)
        for r in range(world):
            if T_per_rank[r]:
                want = oracle.reduce_partials(np.stack(partials[r]))
                assert np.array_equal(st[r]["out"].reshape(T_per_rank[r], H), want), (step, r)
