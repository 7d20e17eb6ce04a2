"""bench.py's expert-parallel modes run on one GPU and print one contract line: the replicated-token
exchange (--ep, dist.EpExchange with one rank) and the token-sharded layer (--a2a, dist.EpAllToAll with
one rank).  Several GPUs run the same code under torchrun; here it is the single-rank form."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("mode", ["--ep", "--a2a"])
def test_expert_parallel_bench_modes(mode):
    proc = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), mode, "--workload", "tiny_T64_E8_k2",
                           "--steps", "5", "--warmup", "3", "--no-cpu-baseline"],
                          capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert proc.returncode == 0, proc.stderr[-3000:]
    lines = [ln for ln in proc.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, lines
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in d, key
    assert d["value"] > 0 and d["scaling"] == "strong" and d["n_gpus"] == 1
    assert d["config"]["workload"] == "tiny_T64_E8_k2"
    assert d["gpu_launches"] > 0


def test_default_bench_line_carries_the_contract_keys():
    """The single-GPU line: roofline of the dominant kernel, the CPU baseline (per stage), the end-to-end
    figure with its copied bytes, clocks and the launch count, on a small workload."""
    proc = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "tiny_T64_E8_k2",
                           "--steps", "5", "--warmup", "3", "--cpu-seconds", "1", "--stage-steps", "5",
                           "--e2e-steps", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert proc.returncode == 0, proc.stderr[-3000:]
    lines = [ln for ln in proc.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, lines
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e",
                "gpu_launches", "clocks"):
        assert key in d, key
    assert d["config"]["workload"] == "tiny_T64_E8_k2" and d["steps"] == 5 and d["warmup"] == 3
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    c = d["cpu_baseline"]
    assert c["kind"] == "oracle" and c["cores"] == 1 and set(c["per_stage_ms"]) == {"topk", "align", "gather", "combine"}
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] == d["launches_per_step"] * d["steps"]
    assert d["workloads"] == []  # a named workload times that workload alone
