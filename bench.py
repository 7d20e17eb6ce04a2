#!/usr/bin/env python
"""Benchmark of the MoE token-routing path (gate + align + permute-gather + combine) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = MoeRouter.step over one batch: moe_route_dispatch (gating + align + permute-gather:
three kernels, or one for decode-sized batches) -> moe_combine (the stand-in expert outputs replace
the expert MLPs between gather and combine), replayed as one CUDA graph.  Inputs are resident in HBM.
The headline is the largest workload (65536 tokens, 256 experts, top-8, hidden 7168, Zipf-skewed
routing); the same run also times the prefill, non-power-of-2 and decode workloads and reports them
under ``workloads`` (the decode workload: every route pattern, the worst one reported).
When one step moves more bytes than L2 holds (the prefill workloads), the K steps are replayed
back to back between one pair of CUDA events on the launching stream; otherwise L2 is flushed (a
256 MiB write, then a 256 MiB read, so no dirty flush lines are written back inside a timed step)
before each step and every step is timed with its own pair of events (``--flush-always`` forces
this mode; the flushed figure is reported beside the other).  The result is the max over ranks.
N > 1 runs the layer expert-parallel (strong scaling): every rank routes the same tokens with its own
contiguous block of E/N experts, combines its local slots into the owners' receive buffers (CUDA IPC,
the stores crossing NVLink) and reduces the rows it owns (dist.EpExchange); a step ends with the
layer output spread over the ranks.  ``--dp`` runs one independent batch per GPU instead (weak
scaling, no exchange); ``--ep`` takes the expert-parallel step on one GPU too; ``--a2a`` shards the
workload's tokens over the ranks instead (dist.EpAllToAll: each owner pulls the hidden rows its
experts need from every rank and pushes each rank's partial combine back).
Rank 0 prints one JSON line.

Also reported: per-stage device times and achieved HBM bandwidth from the algorithmic bytes (for
the step's path and for the four stage entry points),
the roofline of the dominant kernel against the measured copy peak, an end-to-end figure
through MoeRouter.step_from_host (pinned host inputs copied in and the output copied back
inside the timed region, double-buffered over two streams), SM clocks sampled while the workload
is measured, and the CPU oracle timed on this host as a baseline (per stage and in total).
``--impl reference`` times the CPU oracle alone.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "routed tokens/s (gate+align+permute+combine) and achieved HBM GB/s vs ~8 TB/s"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_HBM_GBS = 6650.0
NVLINK_PEER_GBS = 770.0  # measured peer copy on this machine's B200s, per direction per GPU
KERNEL_SOURCES = {
    "topk_row_warp_kernel": "token_dispatch_topk_b200/csrc/topk_softmax.cu",
    "align_cluster_kernel": "token_dispatch_topk_b200/csrc/align_permute.cu",
    "gather_tma_kernel": "token_dispatch_topk_b200/csrc/gather_combine.cu",
    "combine_tma_kernel": "token_dispatch_topk_b200/csrc/gather_combine.cu",
    "combine_small_kernel": "token_dispatch_topk_b200/csrc/gather_combine.cu",
    "gate_count_kernel+tile_scan_kernel+place_gather_kernel": "token_dispatch_topk_b200/csrc/route_fused.cu",
    "gate_count_lanes_kernel+tile_scan_kernel+place_gather_kernel": "token_dispatch_topk_b200/csrc/route_fused.cu",
    "gate_count_kernel+tile_scan_kernel+place_gather_kernel<false>": "token_dispatch_topk_b200/csrc/route_fused.cu",
    "topk_lane_kernel": "token_dispatch_topk_b200/csrc/topk_softmax.cu",
    "align_count_kernel+align_place_kernel": "token_dispatch_topk_b200/csrc/align_permute.cu",
    "route_small_kernel": "token_dispatch_topk_b200/csrc/route_fused.cu",
    "route_decode_kernel": "token_dispatch_topk_b200/csrc/route_fused.cu",
}
STAGE_KERNEL = {"topk": "topk_row_warp_kernel", "align": "align_cluster_kernel", "gather": "gather_tma_kernel",
                "combine": "combine_tma_kernel", "dispatch": "gate_count_kernel+tile_scan_kernel+place_gather_kernel"}


def parse_args():
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=None,
                   help="workload name (default: the skewed 65536-token prefill, with the other workloads as sub-records)")
    p.add_argument("--no-sub-workloads", action="store_true", help="time the headline workload only")
    p.add_argument("--dp", action="store_true", help="N > 1: one independent batch per GPU (no exchange)")
    p.add_argument("--ep", action="store_true", help="the expert-parallel step even on one GPU")
    p.add_argument("--a2a", action="store_true",
                   help="the expert-parallel layer with the tokens sharded over the ranks (EpAllToAll)")
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--no-graph", action="store_true", help="launch the calls directly instead of a graph")
    p.add_argument("--flush-always", action="store_true",
                   help="flush L2 before every timed step even when a step moves more bytes than L2 holds")
    p.add_argument("--stage-steps", type=int, default=None,
                   help="instrumented steps for the per-stage breakdown (default: min(steps, 500))")
    p.add_argument("--e2e-steps", type=int, default=None, help="timed end-to-end steps (default: min(steps, 200))")
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU-oracle baseline budget (rank 0, N=1)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--reference-seconds", type=float, default=150.0, help="--impl reference: total time budget")
    return p.parse_args()


# ------------------------------------------------------------------------- helpers --
def dist_env():
    from token_dispatch_topk_b200.dist import rank_env
    return rank_env()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, burst copy)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s (no MEASURED_PEAKS.json)"


def source_sha(rel: str) -> str:
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source is unchanged since."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            table = json.load(f)
        ent = table[f"{kernel}|{workload}"]
        if ent.get("source_sha256") != source_sha(KERNEL_SOURCES[kernel]):
            return None
        return float(ent["dram_bytes_per_launch"])
    except Exception:
        return None


def algorithmic_bytes(wl, R: int, C: int, NB: int) -> dict:
    """Bytes each stage must move (each input read once, each output written once)."""
    lb = 2 if wl.logits_dtype == "bf16" else 4
    T, E, k, H, El = wl.T, wl.E, wl.k, wl.H, wl.experts_local
    mp = E * 4 if wl.E_local is not None else 0
    return {
        "topk": T * E * lb + T * k * 8,
        "align": 2 * T * k * 4 + mp + C * 4 + NB * 4 + (2 * El + 2) * 4,
        "gather": T * H * 2 + R * H * 2 + T * k * 4,
        "combine": R * H * 2 + T * k * 8 + T * H * 2,
    }


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason sampling in the background (200 ms period)."""
    FIELDS = ("uuid,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "note": "nvidia-smi unavailable"}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [ln.split(",") for ln in self.file.read().splitlines() if ln.strip()]
        os.unlink(self.file.name)
        rows = [[c.strip() for c in r] for r in rows if len(r) >= 10]
        if self.uuid:
            mine = [r for r in rows if self.uuid in r[0]]
            rows = mine or rows
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ CPU oracle leg --
ORACLE_STAGES = ("topk", "align", "gather", "combine")


def oracle_pass(oracle_mod, wl, logits_np, hidden_bits, y_bits, emap_np, t0: int, n: int, times=None):
    """The oracle pipeline on tokens [t0, t0+n) of the workload (gate, align, gather, combine);
    appends each stage's wall time (s) to ``times[stage]`` when given."""
    clk = time.perf_counter
    a = clk()
    w, ids = oracle_mod.topk_softmax(logits_np[t0:t0 + n], wl.k, wl.renormalize)
    b = clk()
    al = oracle_mod.align_permute(ids, wl.E, wl.block_size, emap_np, wl.experts_local)
    c = clk()
    npad = int(al["num_tokens_post_pad"][0])
    oracle_mod.gather(hidden_bits[t0:t0 + n], wl.k, al["sorted_token_ids"], npad, al["capacity"])
    d = clk()
    oracle_mod.combine(y_bits[:al["capacity"]], w, al["inv_perm"])
    e = clk()
    if times is not None:
        for name, dt in zip(ORACLE_STAGES, (b - a, c - b, d - c, e - d)):
            times[name].append(dt)
    return n


def oracle_sample_tokens(wl) -> int:
    """Tokens of the workload in one oracle pass of the CPU baseline (a few seconds of CPU work)."""
    return min(wl.T, 2048 if wl.H > 4096 else 4096)


def host_inputs_numpy(wl, seed: int, T_max: int):
    """The first T_max tokens of the workload as numpy arrays for the oracle (bf16 as uint16 bits).
    The counter-based generator gives the same bits on any device; the large buffers are generated on
    the GPU when there is one (faster) and copied to the host."""
    import numpy as np
    import torch
    from token_dispatch_topk_b200 import inputs as I
    gen = "cuda" if torch.cuda.is_available() else "cpu"
    T = min(wl.T, T_max)
    logits = I.make_logits(wl, seed=seed, T=T)
    logits_np = logits.view(torch.int16).numpy().view(np.uint16) if logits.dtype == torch.bfloat16 else logits.numpy()
    hidden = I.make_hidden(wl, seed=seed, T=T, device=gen).cpu()
    hidden_bits = hidden.view(torch.int16).numpy().view(np.uint16)
    cap = T * wl.k + wl.experts_local * (wl.block_size - 1)
    y = I.make_expert_out(cap, wl.H, seed=seed, device=gen).cpu()
    y_bits = y.view(torch.int16).numpy().view(np.uint16)
    emap = I.expert_map(wl)
    return logits_np, hidden_bits, y_bits, None if emap is None else emap.numpy()


def host_cpu() -> dict:
    """CPU model and logical core count of this host (for the CPU-baseline record)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"model": model, "logical_cores": os.cpu_count()}


def cpu_oracle_rate(wl, seed: int, budget_s: float, runs: int = 5):
    """Tokens/s of the oracle on this host (single-threaded) over a bounded token sample: the median
    over up to `runs` passes (fewer when the budget runs out), per stage and in total."""
    import oracle as oracle_mod
    oracle_mod.default()
    logits_np, hidden_bits, y_bits, emap_np = host_inputs_numpy(wl, seed, oracle_sample_tokens(wl))
    T = logits_np.shape[0]
    times = {s: [] for s in ORACLE_STAGES}
    t_start = time.perf_counter()
    passes = 0
    while passes < runs:
        oracle_pass(oracle_mod, wl, logits_np, hidden_bits, y_bits, emap_np, 0, T, times)
        passes += 1
        if time.perf_counter() - t_start >= budget_s:
            break
    per_stage = {s: statistics.median(v) for s, v in times.items()}
    total = statistics.median([sum(times[s][i] for s in ORACLE_STAGES) for i in range(passes)])
    return {"value": T / total, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"the first {T} tokens of the workload, median of {passes} oracle passes, single thread",
            "per_stage_ms": {s: 1e3 * v for s, v in per_stage.items()}, "total_ms": 1e3 * total,
            "host": host_cpu()}


def run_reference(args, wl):
    """--impl reference: the CPU oracle on this host as the reference arm."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle as oracle_mod
    oracle_mod.default()
    steps, warm = args.steps, args.warmup
    # calibrate the per-step sample so that warmup + steps fit the time budget
    T_cal = min(wl.T, 64)
    logits_np, hidden_bits, y_bits, emap_np = host_inputs_numpy(wl, args.seed, oracle_sample_tokens(wl))
    t = time.perf_counter()
    oracle_pass(oracle_mod, wl, logits_np, hidden_bits, y_bits, emap_np, 0, T_cal)
    per_token = max((time.perf_counter() - t) / T_cal, 1e-7)
    per_step_budget = args.reference_seconds / max(1, steps + warm)
    n = int(max(1, min(logits_np.shape[0], per_step_budget / per_token)))
    for i in range(warm):
        oracle_pass(oracle_mod, wl, logits_np, hidden_bits, y_bits, emap_np, 0, n)
    times = {s: [] for s in ORACLE_STAGES}
    t = time.perf_counter()
    for i in range(steps):
        t0 = (i * n) % max(1, logits_np.shape[0] - n + 1)
        oracle_pass(oracle_mod, wl, logits_np, hidden_bits, y_bits, emap_np, t0, n, times)
    el = time.perf_counter() - t
    value = steps * n / el
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": steps,
            "warmup": warm, "ms_per_step": 1e3 * el / steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64 softmax, fp32 combine", "data": "synthetic",
            "config": {"workload": wl.name, **{k: v for k, v in wl.as_config().items() if k != "name"}},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"{n} tokens of the workload per step, single-threaded C++ oracle",
                             "per_stage_ms": {s: 1e3 * statistics.median(v) for s, v in times.items()},
                             "host": host_cpu()},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------ GPU leg --
class Ctx:
    """What every workload measurement shares: the device, stream, L2 flush buffers, rank info."""

    def __init__(self, args, dev, ws, rank):
        import torch
        self.args, self.dev, self.ws, self.rank = args, dev, ws, rank
        self.stream = torch.cuda.Stream(device=dev)
        self.flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.flush_read = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
        self.l2_bytes = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0) or (126 << 20))
        self.sms = torch.cuda.get_device_properties(dev).multi_processor_count
        self.uuid = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(dev).uuid)
        except Exception:
            pass

    def flush(self, i=0):
        # write a buffer larger than L2, then read another one: L2 is left holding only clean
        # lines of a buffer the step never touches, so no flush write-back lands in a timed step
        self.flush_buf.fill_(i & 0xFF)
        self.flush_read.max()


def stage_kernels(wl, r, sms: int) -> dict:
    """The kernels each entry point launches for this workload (the library's selection rules; the
    lane-gating rule is moe_gate::lane_gating_fits in csrc/gate_lane.cuh)."""
    sk = dict(STAGE_KERNEL)
    elem = 2 if wl.logits_dtype == "bf16" else 4
    lanes = wl.k <= 8 and (wl.E * elem) % 16 == 0 and (
        (wl.E <= 64 and wl.T >= 1024) or (elem == 2 and wl.E <= 256 and wl.T >= 16384))
    if r.small_batch:
        sk["dispatch"] = "route_decode_kernel" if wl.T * wl.k <= 32 else "route_small_kernel"
    elif lanes:
        sk["dispatch"] = "gate_count_lanes_kernel+tile_scan_kernel+place_gather_kernel"
    if lanes:
        sk["topk"] = "topk_lane_kernel"
    P = wl.T * wl.k
    if 4096 < P <= 65536:  # the fused path's tile kernels, placement only
        sk["align"] = "gate_count_kernel+tile_scan_kernel+place_gather_kernel<false>"
    elif P > 65536 or wl.experts_local > 512:  # beyond one cluster: the two-kernel align
        sk["align"] = "align_count_kernel+align_place_kernel"
    if wl.T * (-(-wl.H * 2 // 4096)) < sms:  # fewer 4 KB row chunks than SMs: the small-batch combine
        sk["combine"] = "combine_small_kernel"
    return sk


def measure_workload(wl, ctx: Ctx, headline: bool) -> dict:
    """Time one workload's step on this rank's GPU; the headline also gets e2e, clocks and the CPU baseline."""
    import torch
    import token_dispatch_topk_b200 as tdt
    from token_dispatch_topk_b200 import inputs as I
    from token_dispatch_topk_b200.dist import max_over_ranks, rank_seed

    args, dev, stream, ws, rank = ctx.args, ctx.dev, ctx.stream, ctx.ws, ctx.rank
    seed = rank_seed(args.seed, rank)  # an independent batch per rank
    # ---- inputs resident in HBM (counter-based generator: the same bits as on the host)
    logits = I.make_logits(wl, seed=seed, device=dev)
    hidden = I.make_hidden(wl, seed=seed, device=dev)
    y = I.make_expert_out(wl.capacity, wl.H, seed=seed, device=dev)
    r = tdt.MoeRouter(wl.T, wl.E, wl.k, wl.H, wl.block_size, wl.renormalize, E_local=wl.E_local,
                      expert_map=I.expert_map(wl), logits_dtype=logits.dtype, device=dev)
    flush = ctx.flush
    sampler = ClockSampler(ctx.uuid) if (rank == 0 and headline) else None
    if sampler:
        sampler.start()
        time.sleep(0.4)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for _ in range(3):
            r.step(logits, hidden, y)
    stream.synchronize()
    if r.device_status() != tdt.MOE_OK:
        raise RuntimeError(f"{wl.name}: device status after warm-up steps is not MOE_OK")
    R = int(r.align.counts.sum().item())
    npad = int(r.align.num_tokens_post_pad.item())
    NB = r.align.expert_ids.numel()
    launches_per_step = 2 if r.small_batch else 4  # the decode kernel + combine, or gate_count, tile_scan, place_gather, combine

    use_graph = not args.no_graph
    graphs = {}

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        return g

    if use_graph:
        graphs["step"] = capture(lambda: r.step(logits, hidden, y))
    stage_fns = {"step": lambda: r.step(logits, hidden, y)}

    def run(name):
        if use_graph:
            graphs[name].replay()
        else:
            stage_fns[name]()

    step_samples = {}

    def timed(name, iters, warm):
        """Sum of per-iteration event times (ms), L2 flushed before each iteration."""
        with torch.cuda.stream(stream):
            for i in range(warm):
                flush(i)
                run(name)
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
            for i, (a, b) in enumerate(evs):
                flush(i)
                a.record(stream)
                run(name)
                b.record(stream)
        stream.synchronize()
        per_step = [a.elapsed_time(b) for a, b in evs]
        step_samples[name] = per_step
        return sum(per_step)

    def timed_back_to_back(name, iters, warm):
        """Time (ms) of `iters` steps replayed back to back between one pair of events (no flush:
        used when one step's bytes exceed L2, so no step finds its inputs left there by the last)."""
        with torch.cuda.stream(stream):
            for i in range(warm):
                run(name)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for i in range(iters):
                run(name)
            b.record(stream)
        stream.synchronize()
        return a.elapsed_time(b)

    abytes = algorithmic_bytes(wl, R, r.capacity, NB)
    step_bytes = abytes["topk"] + abytes["align"] + abytes["gather"] + abytes["combine"]
    back_to_back = step_bytes > ctx.l2_bytes and not args.flush_always

    # ---- the timed region: K steps
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    t_region = time.perf_counter()
    if back_to_back:
        total_ms = timed_back_to_back("step", args.steps, args.warmup)
    else:
        total_ms = timed("step", args.steps, args.warmup)
    torch.cuda.synchronize()
    t_region = time.perf_counter() - t_region
    total_ms = max_over_ranks(total_ms, dev)
    if ws > 1:
        dist.barrier()
    ms_per_step = total_ms / args.steps
    value = ws * wl.T * args.steps / (total_ms / 1e3)
    # the same step with L2 flushed before each step and events around each step (adds the
    # launch-to-event latency of a lone graph, about 5 us, to every step)
    n_fl = min(args.steps, 200)
    flushed_ms_per_step = (timed("step", n_fl, 3) / n_fl) if back_to_back else ms_per_step
    qs = statistics.quantiles(step_samples["step"], n=10) if len(step_samples.get("step", [])) >= 10 else None
    flushed_pct_us = None if qs is None else {"p10": 1e3 * qs[0], "p50": 1e3 * statistics.median(step_samples["step"]),
                                              "p90": 1e3 * qs[-1], "steps": len(step_samples["step"])}

    # ---- per-stage times inside the step, and roofline
    # The step is captured once more with external event records between its stages, so each
    # stage is timed on the launching stream as it runs inside a step (same flush protocol).  The
    # fused step has two stages (dispatch = gate_count + place_gather kernels, then combine); the
    # four stage entry points are timed the same way for comparison.
    peak, peak_src = measured_peaks()
    abytes["dispatch"] = abytes["topk"] + abytes["align"] + abytes["gather"]
    st_iters = args.stage_steps or min(args.steps, 500)
    stage_kernel = stage_kernels(wl, r, ctx.sms)

    def stage_times(names, calls):
        marks = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(names) + 1)]

        def instrumented():
            marks[0].record()
            for i, fn in enumerate(calls):
                fn()
                marks[i + 1].record()

        if use_graph:
            g_inst = capture(instrumented)
        sums = [0.0] * len(names)
        warm = min(args.warmup, 10)
        with torch.cuda.stream(stream):
            for i in range(warm + st_iters):
                flush(i)
                if use_graph:
                    g_inst.replay()
                else:
                    instrumented()
                stream.synchronize()
                if i >= warm:
                    for j in range(len(names)):
                        sums[j] += marks[j].elapsed_time(marks[j + 1])
        if use_graph:
            del g_inst
        out = {}
        for j, name in enumerate(names):
            ms = sums[j] / st_iters
            out[name] = {"us": 1e3 * ms, "algorithmic_bytes": abytes[name],
                         "achieved_gbs": abytes[name] / (ms * 1e-3) / 1e9, "kernel": stage_kernel[name],
                         "timing": "CUDA events between the stages of the step graph"}
        return out

    stages = stage_times(ORACLE_STAGES, [lambda: r.gate(logits), lambda: r.align_permute(),
                                         lambda: r.gather(hidden, hidden_ready=True), lambda: r.combine(y)])
    stages_fused = stage_times(("dispatch", "combine"), [lambda: r.dispatch(logits, hidden), lambda: r.combine(y)])

    # the dominant single kernel of the step: the combine (about half of the bytes) above the
    # small-batch limits; for small batches the longer of the step's two kernels.  Its launch time
    # is measured without the per-step event floor: a graph of n x [L2 flush, launch] minus a graph
    # of n x [L2 flush], both replayed between one pair of events on the launching stream.
    def launch_us(fn, n=20, reps=5):
        def both():
            for i in range(n):
                flush(i)
                fn()

        def flush_only():
            for i in range(n):
                flush(i)

        ga, gb = capture(both), capture(flush_only)
        res = []
        with torch.cuda.stream(stream):
            for g in (ga, gb):
                g.replay()
                ts = []
                for _ in range(reps):
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    g.replay()
                    e1.record(stream)
                    ts.append((e0, e1))
                stream.synchronize()
                res.append(statistics.median(a.elapsed_time(b) for a, b in ts))
        del ga, gb
        return 1e3 * (res[0] - res[1]) / n

    in_step = stages_fused
    dom = max(in_step, key=lambda n: in_step[n]["us"]) if r.small_batch else "combine"
    dom_fn = (lambda: r.combine(y)) if dom == "combine" else (lambda: r.dispatch(logits, hidden))
    dom_us = launch_us(dom_fn)
    ach = abytes[dom] / (dom_us * 1e-6) / 1e9
    roofline = {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                "traffic": ncu_traffic(stage_kernel[dom], wl.name), "kernel": stage_kernel[dom],
                "peak_source": peak_src, "launch_us": dom_us,
                "timing": "graph of 20 x [L2 flush, launch] minus graph of 20 x [L2 flush], per launch",
                "algorithmic_bytes_per_launch": abytes[dom]}

    # ---- injected route patterns of the decode workload: the step for routes given by the caller
    # (align + permute-gather + combine), one graph per pattern, same flush protocol; worst reported
    patterns = None
    if wl.name.startswith("ep_decode"):
        w_inj = I.decode_pattern_weights(seed=seed).to(dev)
        pat_us, device = {}, {}
        for pname in I.DECODE_PATTERNS:
            ids_p = I.decode_pattern_ids(pname).to(dev)
            fn = (lambda ids_p=ids_p: r.step_routes(ids_p, w_inj, hidden, y))
            if use_graph:
                graphs["pattern"] = capture(fn)
            stage_fns["pattern"] = fn
            n_it = min(args.steps, 500)
            pat_us[pname] = 1e3 * timed("pattern", n_it, min(args.warmup, 10)) / n_it
            device[pname] = launch_us(fn)
        device["logits"] = launch_us(lambda: r.step(logits, hidden, y))
        patterns = {"us_per_step": pat_us, "worst_us": max(pat_us.values()),
                    "worst": max(pat_us, key=pat_us.get),
                    "device_us_per_step": device, "device_worst_us": max(device.values()),
                    "device_worst": max(device, key=device.get),
                    "device_timing": "graph of 20 x [L2 flush, step] minus graph of 20 x [L2 flush], per step "
                                     "(kernels and the gaps between them, without the per-step event latency)",
                    "path": "MoeRouter.step_routes: moe_route_dispatch (given routes) + moe_combine, one graph each"}
        if r.device_status() != tdt.MOE_OK:
            raise RuntimeError("device status after the route-pattern steps is not MOE_OK")

    total_bytes = step_bytes
    rec = {
        "workload": wl.name, "T": wl.T, "E": wl.E, "E_local": wl.experts_local, "k": wl.k, "H": wl.H,
        "value": value, "unit": UNIT, "ms_per_step": ms_per_step,
        "achieved_hbm_gbs": total_bytes / (ms_per_step * 1e-3) / 1e9,
        "algorithmic_bytes_per_step": total_bytes,
        "hbm_frac_of_8tbs": total_bytes / (ms_per_step * 1e-3) / 8e12,
        "hbm_frac_of_measured_peak": total_bytes / (ms_per_step * 1e-3) / 1e9 / peak,
        "routed_slots_local": R, "num_tokens_post_pad": npad,
        "l2": (f"not flushed: steps replayed back to back, each moving {step_bytes / 2**20:.0f} MiB "
               f"> L2 ({ctx.l2_bytes >> 20} MiB)") if back_to_back else
              (f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write + "
               f"{L2_FLUSH_BYTES >> 20} MiB read of another buffer)"),
        "flushed_ms_per_step": flushed_ms_per_step, "flushed_step_us_percentiles": flushed_pct_us,
        "step_path": "moe_route_dispatch (single kernel) + moe_combine" if r.small_batch else
                     "moe_route_dispatch (three kernels) + moe_combine",
        "roofline": roofline, "stages": stages_fused, "stages_four_call_path": stages,
        "decode_route_patterns": patterns, "launches_per_step": launches_per_step,
        "timed_region_s": t_region,
    }

    if headline:
        # ---- end to end through the public API, from pinned host buffers (double-buffered: the next
        # step's host->device copies and the previous step's device->host copy overlap the step)
        e2e_steps = args.e2e_steps or min(args.steps, 200)
        logits_h = logits.cpu().pin_memory()
        hidden_h = hidden.cpu().pin_memory()
        outs_h = [torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        pipe = tdt.HostStepPipeline(r, expert_out=y)
        for i in range(3):
            pipe.submit(logits_h, hidden_h, outs_h[i % 2])
        pipe.synchronize()
        e0, e1 = pipe.timed(lambda i: pipe.submit(logits_h, hidden_h, outs_h[i % 2]), e2e_steps)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
        h2d = logits_h.numel() * logits_h.element_size() + hidden_h.numel() * hidden_h.element_size()
        d2h = outs_h[0].numel() * outs_h[0].element_size()
        rec["e2e"] = {"value": ws * wl.T * e2e_steps / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h, "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps,
                      "api": "HostStepPipeline over MoeRouter (pinned H2D of logits+hidden on one copy stream, "
                             "moe_route_dispatch + moe_combine, D2H of out on another; two buffer sets)"}
        del pipe
        if r.device_status() != tdt.MOE_OK:
            raise RuntimeError("device status after the timed steps is not MOE_OK")
        rec["clocks"] = sampler.stop() if sampler else None
        if rec["clocks"] is not None:
            rec["clocks"]["window"] = ("sampled every 200 ms from before the warm-up steps to the end of the "
                                       "end-to-end steps (timed steps, per-stage and per-launch timing inside)")
        rec["gpu_launches"] = launches_per_step * args.steps
        if rank == 0 and ws == 1 and not args.no_cpu_baseline:
            rec["cpu_baseline"] = cpu_oracle_rate(wl, seed, args.cpu_seconds)
    elif rank == 0 and ws == 1 and not args.no_cpu_baseline:
        rec["cpu_baseline"] = cpu_oracle_rate(wl, seed, min(3.0, args.cpu_seconds))  # per stage, a shorter budget
    del graphs
    if r.device_status() != tdt.MOE_OK:
        raise RuntimeError(f"{wl.name}: device status at the end is not MOE_OK")
    return rec


def measure_ep(wl, ctx: Ctx) -> dict:
    """The expert-parallel layer step over the ranks (strong scaling): every rank routes the same T tokens
    with its own block of experts (moe_route_dispatch), combines its local slots into the owners'
    receive buffers and reduces the rows it owns (dist.EpExchange: a stream synchronisation and a
    process-group barrier inside every step, so no CUDA graph).  Timed with CUDA events on the
    launching stream around K steps, max over ranks; value = T * K / that time."""
    import torch
    import torch.distributed as dist
    import token_dispatch_topk_b200 as tdt
    from token_dispatch_topk_b200 import inputs as I
    from token_dispatch_topk_b200.dist import EpExchange, ep_expert_map, max_over_ranks

    args, dev, stream, ws, rank = ctx.args, ctx.dev, ctx.stream, ctx.ws, ctx.rank
    emap, El = ep_expert_map(wl.E, ws, rank)
    logits = I.make_logits(wl, seed=args.seed, device=dev)  # the same tokens on every rank
    hidden = I.make_hidden(wl, seed=args.seed, device=dev)
    r = tdt.MoeRouter(wl.T, wl.E, wl.k, wl.H, wl.block_size, wl.renormalize, E_local=El, expert_map=emap,
                      logits_dtype=logits.dtype, device=dev)
    y = I.make_expert_out(r.capacity, wl.H, seed=args.seed * 16 + 5 + rank, device=dev)  # this rank's experts
    ex = EpExchange(wl.T, wl.H, dev)

    def step():
        r.dispatch(logits, hidden, stream=stream)
        ex.combine_reduce(y, r.topk_weights, r.align.inv_perm, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
    stream.synchronize()
    if r.device_status() != tdt.MOE_OK:
        raise RuntimeError("expert-parallel warm-up: device status is not MOE_OK")
    sampler = ClockSampler(ctx.uuid) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.4)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
    stream.synchronize()
    total_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    # end to end: the step's inputs copied in from pinned host memory, this owner's rows copied out
    logits_h, hidden_h = logits.cpu().pin_memory(), hidden.cpu().pin_memory()
    lo, hi = ex.ranges[rank]
    out_h = torch.empty((hi - lo, wl.H), dtype=torch.bfloat16).pin_memory()
    e2e_steps = args.e2e_steps or min(args.steps, 200)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        f0.record(stream)
        for _ in range(e2e_steps):
            r.logits_dev.copy_(logits_h, non_blocking=True)
            r.hidden_dev.copy_(hidden_h, non_blocking=True)
            r.dispatch(r.logits_dev, r.hidden_dev, stream=stream)
            out = ex.combine_reduce(y, r.topk_weights, r.align.inv_perm, stream=stream)
            out_h.copy_(out, non_blocking=True)
        f1.record(stream)
    stream.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), dev)
    clocks = sampler.stop() if sampler else None
    if r.device_status() != tdt.MOE_OK:
        raise RuntimeError("expert-parallel steps: device status is not MOE_OK")
    R = int(r.align.counts.sum().item())
    nvlink_bytes = sum((b - a) * wl.H * 2 for o, (a, b) in enumerate(ex.ranges) if o != rank)
    # kernels per step: the dispatch (one kernel for decode-sized batches; else gating, tile scan and
    # placement), one combine per owner with tokens, one reduce on an owner with tokens
    n_dispatch = 1 if r.small_batch else 3
    per_step = n_dispatch + sum(1 for a, b in ex.ranges if b > a) + (1 if hi > lo else 0)
    step_s = total_ms / args.steps / 1e3
    # roofline of the exchange: the bytes this rank's combine stores into other ranks' memory, against the
    # measured peer-copy bandwidth of this machine (770 GB/s per direction per GPU; 900 GB/s nominal)
    nvlink = None if nvlink_bytes == 0 else {
        "bound": "nvlink", "bytes_per_step": nvlink_bytes, "peak": NVLINK_PEER_GBS, "unit": "GB/s",
        "achieved": nvlink_bytes / step_s / 1e9, "frac": nvlink_bytes / step_s / 1e9 / NVLINK_PEER_GBS,
        "target_ms_per_step": 1e3 * nvlink_bytes / (NVLINK_PEER_GBS * 1e9),
        "note": "achieved = this rank's peer-store bytes over the whole step time (the step also gates, "
                "gathers and reduces)"}
    return {"workload": wl.name, "value": wl.T * args.steps / (total_ms / 1e3), "unit": UNIT,
            "ms_per_step": total_ms / args.steps, "E_local": El, "routed_slots_local_rank0": R,
            "owned_tokens_rank0": hi - lo, "peer_store_bytes_per_rank_per_step": nvlink_bytes,
            "nvlink_roofline": nvlink,
            "launches_per_step": per_step, "gpu_launches": per_step * args.steps, "clocks": clocks,
            "e2e": {"value": wl.T * e2e_steps / (e2e_ms / 1e3), "unit": UNIT,
                    "h2d_bytes_per_step": logits_h.numel() * logits_h.element_size() +
                    hidden_h.numel() * hidden_h.element_size(),
                    "d2h_bytes_per_step": out_h.numel() * out_h.element_size(), "steps": e2e_steps,
                    "api": "MoeRouter.dispatch + EpExchange.combine_reduce, pinned H2D of logits and hidden, "
                           "D2H of this owner's rows (rank 0's bytes)"},
            "parallelism": f"expert parallel over {ws} ranks ({El} local experts each): moe_route_dispatch, "
                           f"moe_combine into the owners' receive buffers (CUDA IPC), barrier, moe_reduce_partials",
            "timing": "CUDA events around K steps on the launching stream (host barrier inside each step), "
                      "max over ranks"}


def measure_a2a(wl, ctx: Ctx) -> dict:
    """The expert-parallel layer with the workload's T tokens sharded over the ranks (dist.EpAllToAll,
    strong scaling): rank r gates its own token range; every owner aligns every rank's routes on its
    experts, pulls the hidden rows it needs and pushes each rank's partial combine back; each rank
    reduces its partials.  Two barriers per step (no CUDA graph).  CUDA events around K steps on the
    launching stream, max over ranks; value = T * K / that time."""
    import torch
    import torch.distributed as dist
    import token_dispatch_topk_b200 as tdt
    from token_dispatch_topk_b200 import inputs as I
    from token_dispatch_topk_b200.dist import EpAllToAll, ep_token_range, max_over_ranks

    args, dev, stream, ws, rank = ctx.args, ctx.dev, ctx.stream, ctx.ws, ctx.rank
    ranges = [ep_token_range(wl.T, ws, r) for r in range(ws)]
    lo, hi = ranges[rank]
    T_per_rank = [b - a for a, b in ranges]
    logits = I.make_logits(wl, seed=args.seed, device=dev)[lo:hi].contiguous()  # this rank's tokens
    ex = EpAllToAll(T_per_rank, wl.E, wl.k, wl.H, wl.block_size, wl.renormalize, dev, logits_dtype=logits.dtype)
    ex.hidden[:hi - lo].copy_(I.hidden_rows(torch.arange(lo, hi), wl.H, seed=args.seed, device=dev))
    y = I.make_expert_out(ex.capacity, wl.H, seed=args.seed * 16 + 5 + rank, device=dev)  # this owner's experts

    def step():
        ex.step(logits, y, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            step()
    stream.synchronize()
    if tdt.moe_read_status(ex.workspace) != tdt.MOE_OK:
        raise RuntimeError("all-to-all warm-up: device status is not MOE_OK")
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
    stream.synchronize()
    total_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    if tdt.moe_read_status(ex.workspace) != tdt.MOE_OK:
        raise RuntimeError("all-to-all steps: device status is not MOE_OK")
    # kernels per step: gating of this rank's tokens; the align of every rank's routes (one cluster kernel
    # up to 4096 slots, the three tile kernels up to 65536, count + place above or past 512 local experts);
    # a gather and a combine per rank with tokens; the reduce of this rank's rows
    P = wl.T * wl.k
    n_align = 3 if 4096 < P <= 65536 else (1 if P <= 4096 and ex.E_local <= 512 else 2)
    own = 1 if hi > lo else 0
    per_step = own + n_align + 2 * sum(1 for t in T_per_rank if t) + own
    return {"workload": wl.name, "value": wl.T * args.steps / (total_ms / 1e3), "unit": UNIT,
            "ms_per_step": total_ms / args.steps, "E_local": ex.E_local, "tokens_rank0": T_per_rank[0],
            "launches_per_step": per_step, "gpu_launches": per_step * args.steps,
            "parallelism": f"expert parallel over {ws} ranks, tokens sharded ({T_per_rank[0]} on rank 0): gating, "
                           f"align of every rank's routes, moe_gather pulling rows from each rank, moe_combine "
                           f"pushing partials, barrier, moe_reduce_partials",
            "timing": "CUDA events around K steps on the launching stream (host barriers inside each step), "
                      "max over ranks"}


TARGETS = {  # end-to-end targets: fraction of 8 TB/s, or device time of the worst decode route pattern
    "qwen3moe_prefill_T4096_E128_k8": ("hbm_frac_of_8tbs", 0.70),
    "nonpow2_T16384_E60_k4": ("hbm_frac_of_8tbs", 0.70),
    "zipf_prefill_T65536_E256_k8_H7168": ("hbm_frac_of_8tbs", 0.70),
    "ep_decode_T2_E160_local40_k6": ("device_worst_us", 10.0),
}


def target_status(rec: dict):
    t = TARGETS.get(rec["workload"])
    if t is None:
        return None
    key, bar = t
    if key == "device_worst_us":
        v = rec["decode_route_patterns"]["device_worst_us"]
        return {"device_worst_us": v, "bar_us": bar, "met": v < bar}
    return {key: rec[key], "bar": bar, "met": rec[key] >= bar}


def main():
    args = parse_args()
    from token_dispatch_topk_b200 import inputs as I
    wl = I.WORKLOADS[args.workload or I.DEFAULT_WORKLOAD]
    if args.impl == "reference":
        return run_reference(args, wl)

    import torch
    import torch.distributed as dist
    import token_dispatch_topk_b200 as tdt

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))
    tdt.load_library()
    ctx = Ctx(args, dev, ws, rank)

    if args.a2a:
        rec = measure_a2a(wl, ctx)
        if rank == 0:
            print(json.dumps({
                "metric": METRIC, "value": rec["value"], "unit": UNIT, "n_gpus": ws, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded, counter-based; see token_dispatch_topk_b200/inputs.py)",
                "config": {"workload": wl.name, **{k: v for k, v in wl.as_config().items() if k != "name"},
                           "parallelism": rec["parallelism"], "cuda_graph": False},
                "expert_parallel_all_to_all": rec, "gpu_launches": rec["gpu_launches"], "e2e": None,
                "cpu_baseline": None}), flush=True)
        if ws > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    if (ws > 1 and not args.dp) or args.ep:
        rec = measure_ep(wl, ctx)
        if rank == 0:
            print(json.dumps({
                "metric": METRIC, "value": rec["value"], "unit": UNIT, "n_gpus": ws, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded, counter-based; see token_dispatch_topk_b200/inputs.py)",
                "config": {"workload": wl.name, **{k: v for k, v in wl.as_config().items() if k != "name"},
                           "parallelism": rec["parallelism"], "cuda_graph": False},
                "expert_parallel": rec, "gpu_launches": rec["gpu_launches"], "clocks": rec["clocks"],
                "e2e": rec["e2e"], "cpu_baseline": None}), flush=True)
        if ws > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    head = measure_workload(wl, ctx, headline=True)
    head["target"] = target_status(head)
    subs = []
    if args.workload is None and not args.no_sub_workloads:
        torch.cuda.empty_cache()
        for name in I.BENCH_SUB_WORKLOADS:
            rec = measure_workload(I.WORKLOADS[name], ctx, headline=False)
            rec["target"] = target_status(rec)
            subs.append(rec)
            torch.cuda.empty_cache()

    if rank == 0:
        line = {
            "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "dtype_detail": "bf16 activations, fp32 gating math and combine accumulation, int32 indices",
            "data": "synthetic (seeded, counter-based; see token_dispatch_topk_b200/inputs.py)",
            "config": {"workload": wl.name, **{k: v for k, v in wl.as_config().items() if k != "name"},
                       "l2": head["l2"], "cuda_graph": not args.no_graph,
                       "parallelism": "one independent batch per GPU (--dp)" if ws > 1 else "single GPU"},
            **{k: head[k] for k in ("achieved_hbm_gbs", "algorithmic_bytes_per_step", "hbm_frac_of_8tbs",
                                    "hbm_frac_of_measured_peak", "routed_slots_local", "num_tokens_post_pad",
                                    "flushed_ms_per_step", "flushed_step_us_percentiles", "step_path", "roofline",
                                    "stages", "stages_four_call_path", "decode_route_patterns", "target",
                                    "timed_region_s")},
            "e2e": head["e2e"], "cpu_baseline": head.get("cpu_baseline"),
            "gpu_launches": head["gpu_launches"], "launches_per_step": head["launches_per_step"],
            "clocks": head["clocks"],
            "workloads": subs,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
