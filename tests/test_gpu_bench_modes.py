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
