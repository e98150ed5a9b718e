"""The FA_DEBUG_BOUNDS build: every computed global index checked against the extent the kernel's
arguments give its buffer, a failed check recorded in the device status word and the access
skipped (never a fault).  The mechanism is checked on a kernel whose guarded stores stay inside
their buffer; then the bounds-checked library runs small ragged cases through every entry point
with no check failing and outputs identical to the ordinary build's."""
import os
import re
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "quantized_attention_amax_b200", "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def test_failed_check_records_and_skips(tmp_path):
    exe = str(tmp_path / "bounds_check")
    src = os.path.join(HERE, "gpu_progs", "bounds_check.cu")
    subprocess.run([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-I", CSRC, src, "-o",
                    exe], check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    m = re.search(r"status (\d+) stored (\d+) guard (\d+)", r.stdout)
    assert m, r.stdout
    status, stored, guard = map(int, m.groups())
    assert status == (9 << 8) | 2  # the site, then kStatusBounds
    assert stored == 32 and guard == 0


def test_bounds_build_runs_every_entry_point_clean(tmp_path):
    from quantized_attention_amax_b200 import build
    build.build()
    build.build(bounds=True)
    outs = {}
    for lib in ("bounds", "release"):
        env = dict(os.environ)
        if lib == "bounds":
            env["FAQ_LIB"] = "bounds"
        else:
            env.pop("FAQ_LIB", None)
        path = str(tmp_path / f"{lib}.npz")
        r = subprocess.run([sys.executable, os.path.join(HERE, "_bounds_cases.py"), path], capture_output=True,
                           text=True, timeout=600, env=env, cwd=ROOT)
        assert r.returncode == 0, r.stdout + r.stderr  # FA_ERR_BOUNDS would raise here
        outs[lib] = dict(np.load(path))
    assert outs["bounds"].keys() == outs["release"].keys()
    for name in outs["release"]:
        assert np.array_equal(outs["bounds"][name], outs["release"][name], equal_nan=True), name
