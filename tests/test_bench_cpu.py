"""bench.py's command-line contract on a host without a GPU.

The reference arm (the oracle, timed on the host cores) runs on rank 0 only and prints one JSON
line with the arm's own metric, config and cpu_baseline.  Every other rank exits 0 without work.
The library's own arm refuses to run without a CUDA device: it has no CPU fallback.
"""
import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(args, rank=0, world=1):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                          env=env, cwd=ROOT, timeout=600)


def test_reference_arm_prints_one_line_on_rank_zero():
    r = run_bench(["--impl", "reference", "--steps", "2", "--warmup", "1", "--workload", "int8_tiny"], 0, 2)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["steps"] == 2 and d["warmup"] == 1 and d["higher_is_better"] is True
    assert d["config"]["workload"].startswith("int8_tiny")
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_without_work():
    r = run_bench(["--impl", "reference", "--steps", "2", "--warmup", "1"], 1, 2)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a CUDA device")
def test_library_arm_fails_without_a_gpu():
    r = run_bench(["--steps", "3", "--warmup", "3", "--no-supplemental", "--no-cpu-baseline", "--no-e2e"])
    assert r.returncode != 0
    assert "no CUDA device" in r.stdout
