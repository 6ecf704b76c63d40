"""GPU: bench.py's JSON line on a short run of the tiny workload.

The benchmark's own contract, checked where it runs: one JSON line with the
metric, the whole-job value, the timing fields, the roofline object of the
dominant kernel, the end-to-end number with the bytes it copies, the
clocks sampled during the timed region, the launch count, and the oracle's
CPU baseline. Launched by torch.distributed.run with one process, the bench
runs its multi-rank code: a one-rank NCCL group, the double-buffered dW and its
all-reduce on a communication stream, in the timed loop and in the end-to-end
loop.
"""

import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_line_contract():
    out = subprocess.run([sys.executable, "bench.py", "--workload", "tiny", "--steps", "6",
                          "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    lines = [json.loads(x) for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = lines[0]
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "ms_per_step_median", "step_ms", "higher_is_better", "scaling", "vs_baseline",
              "dtype", "precision", "data", "config", "roofline", "kernels", "gpu_launches",
              "clocks", "e2e", "cpu_baseline"):
        assert k in d, k
    assert d["unit"] == "tokens/s" and d["value"] > 0 and d["n_gpus"] == 1
    assert d["steps"] == 6 and d["warmup"] == 3 and len(d["step_ms"]) == 6
    assert "precision" not in d["config"] and d["config"]["workload"].startswith("tiny")
    r = d["roofline"]
    assert r["bound"] in ("tensor", "hbm") and r["achieved"] > 0 and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert d["gpu_launches"] == 9 * 6  # per step: build 2, forward 5, backward 2
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["clocks"] and d["clocks"]["samples"] >= 1
    c = d["cpu_baseline"]
    assert c["kind"] == "oracle" and c["cores"] >= 1 and c["value"] > 0


def test_bench_under_torchrun_runs_the_gradient_sync():
    out = subprocess.run(
        [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "1",
         "--master-addr", "127.0.0.1", "--master-port", "29517", "bench.py", "--workload",
         "tiny", "--steps", "6", "--warmup", "3", "--no-cpu-baseline"],
        cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    lines = [json.loads(x) for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = lines[0]
    assert d["n_gpus"] == 1 and d["value"] > 0 and len(d["step_ms"]) == 6
    assert "all-reduced" in d["config"]["parallelism"]
    a = d["dp_allreduce"]
    assert a["bytes"] > 0 and a["avg_ms"] is not None and a["avg_ms"] >= 0
    assert d["e2e"]["value"] > 0
