"""The FP8 quantizers divide by the scale as x * r plus one FMA correction (quant_common.cuh)
instead of IEEE division.  This compiles a sweep over every bf16 amax and every bf16 |x| <= amax
against the product header and requires the same E4M3 code as IEEE division everywhere."""
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
    m = re.search(r"fast rows (\d+) mismatches (\d+)", r.stdout)
    assert m, r.stdout
    assert int(m.group(1)) > 26000  # nearly every scale takes the fast path
    assert int(m.group(2)) == 0
