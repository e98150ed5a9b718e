"""The quantizers divide by the scale as x * r plus one FMA correction (quant_common.cuh) instead of
IEEE division.  This compiles a sweep against the product header -- every bf16 amax, and every bf16
x with |x| <= amax (dynamic FP8) or every finite bf16 x (static FP8, INT8) -- and requires the same
E4M3 / INT8 code as IEEE division everywhere."""
import os
import re
import subprocess

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "quantized_attention_amax_b200", "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def test_fp8_div_matches_ieee_division_exhaustively(tmp_path):
    exe = str(tmp_path / "fp8_div_exhaustive")
    src = os.path.join(HERE, "gpu_progs", "fp8_div_exhaustive.cu")
    subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-I", CSRC, src, "-o",
                    exe], check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    found = re.findall(r"mode (\d) fast rows (\d+) mismatches (\d+)", r.stdout)
    assert [int(m) for m, _, _ in found] == [0, 1, 2, 3, 4], r.stdout
    for _, fast, bad in found:
        assert int(fast) > 26000  # nearly every scale takes the fast path
        assert int(bad) == 0
