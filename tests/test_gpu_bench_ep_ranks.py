"""bench.py's multi-rank expert-parallel measurements (measure_ep, measure_a2a) run as two ranks, i.e. two
processes, on one GPU with a gloo process group.

On several GPUs, `torchrun --nproc-per-node N bench.py --gpus N` runs these same functions over NCCL,
one GPU per rank. Here both ranks share GPU 0. The receive buffers and hidden rows travel between the
processes through CUDA IPC, exactly as between GPUs. No kernel waits for another process's kernel: every
cross-rank wait is a host barrier. The test checks the plumbing that a multi-GPU run depends on:
- the barriers in warm-up, timing and the end-to-end loop;
- the max-over-ranks timing;
- the record's fields;
- that the device status stays MOE_OK on every rank.
"""
import importlib.util
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, mode, workload, q):
    from datetime import timedelta

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK="0")
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    try:
        spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
        bench = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(bench)
        sys.argv = ["bench.py", "--gpus", str(world), "--steps", "5", "--warmup", "3", "--e2e-steps", "3",
                    "--workload", workload]
        args = bench.parse_args()
        import token_dispatch_topk_b200 as tdt
        from token_dispatch_topk_b200 import inputs as I
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        tdt.load_library()
        ctx = bench.Ctx(args, dev, world, rank)
        wl = I.WORKLOADS[workload]
        rec = bench.measure_ep(wl, ctx) if mode == "ep" else bench.measure_a2a(wl, ctx)
        keep = {k: rec.get(k) for k in ("value", "ms_per_step", "parallelism", "gpu_launches")}
        keep["e2e"] = rec.get("e2e")
        q.put((rank, keep))
        dist.barrier()
    except Exception as exc:  # report instead of hanging the other rank's queue read
        q.put((rank, {"error": repr(exc)}))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode,workload", [("ep", "tiny_T64_E8_k2"), ("ep", "ep_decode_T2_E160_local40_k6"),
                                           ("a2a", "tiny_T64_E8_k2")],
                         ids=["exchange_tiny", "exchange_decode", "all_to_all_tiny"])
def test_bench_expert_parallel_two_ranks_one_gpu(mode, workload):
    assert torch.cuda.is_available()
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, mode, workload, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=120)
    for r in range(world):
        assert "error" not in res[r], res[r]
    for p in procs:
        assert p.exitcode == 0
    # max over ranks: both ranks report the same step time
    assert res[0]["ms_per_step"] == res[1]["ms_per_step"]
    assert res[0]["ms_per_step"] > 0 and res[0]["value"] > 0
    assert f"over {world} ranks" in res[0]["parallelism"]
    if mode == "ep":
        assert res[0]["gpu_launches"] > 0
        e2e = res[0]["e2e"]
        assert e2e["value"] > 0 and e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
