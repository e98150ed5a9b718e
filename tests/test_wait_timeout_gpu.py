"""Failure detection without a GPU fault: every mbarrier wait in the kernels goes through the
bounded wait of sm100.cuh.  This compiles a program against that header with a 2 ms bound, makes
one CTA wait on an mbarrier that nothing arrives at, and checks that every thread gives up, that
the status word holds the waiting site and the timeout code, that the CTA's abort flag is raised,
and that the next kernel runs normally."""
import os
import re
import subprocess

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "quantized_attention_amax_b200", "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def test_bounded_wait_runs_out_and_reports(tmp_path):
    exe = str(tmp_path / "wait_timeout")
    src = os.path.join(HERE, "gpu_progs", "wait_timeout.cu")
    subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-I", CSRC, src, "-o",
                    exe], check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    m = re.search(r"status (\d+) done (\d+) gaveup (\d+) abort (\d+) after (\d+)", r.stdout)
    assert m, r.stdout
    status, done, gaveup, abort, after = map(int, m.groups())
    assert status == (7 << 8) | 1   # the waiting site, then kStatusTimeout
    assert done == 0 and gaveup == 64
    assert abort == 1
    assert after == 64
