"""Build libfaq.so (the C-ABI library) from csrc/*.cu for sm_100a, in-tree.

    python -m quantized_attention_amax_b200.build [--force] [-v] [--bounds]

--bounds builds libfaq_bounds.so instead, with FA_DEBUG_BOUNDS: every computed global index is
checked against the extent the kernel's arguments give its buffer, a failed check is recorded in
the device status word (fa_check_device_status -> FA_ERR_BOUNDS) and the access skipped.  The
package loads it when FAQ_LIB=bounds.

Each .cu compiles to an object under _build/ (in parallel), then one link
step produces quantized_attention_amax_b200/libfaq.so.  nvcc cross-compiles
without a GPU.  The runtime is linked statically; the driver API is reached
through cudaGetDriverEntryPoint, so the library loads on a host without a
GPU driver (the symbol-export tests rely on that).
"""
from __future__ import annotations

import concurrent.futures
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libfaq.so")
BUILD_BOUNDS = os.path.join(PKG, "_build_bounds")
LIB_BOUNDS = os.path.join(PKG, "libfaq_bounds.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
                "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cu"))


def headers():
    hs = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    hs.append(os.path.join(INCLUDE, "faq.h"))
    return hs


def _newest(paths):
    return max(os.path.getmtime(p) for p in paths)


def _compile(src: str, verbose: bool, bounds: bool = False) -> str:
    obj = os.path.join(BUILD_BOUNDS if bounds else BUILD, os.path.basename(src)[:-3] + ".o")
    if os.path.exists(obj) and os.path.getmtime(obj) >= max(os.path.getmtime(src), _newest(headers())):
        return obj
    cmd = [NVCC] + FLAGS + (["-DFA_DEBUG_BOUNDS"] if bounds else []) + (["-Xptxas", "-v"] if verbose else []) + \
        ["-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose:
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, verbose: bool = False, bounds: bool = False) -> str:
    bdir, lib = (BUILD_BOUNDS, LIB_BOUNDS) if bounds else (BUILD, LIB)
    os.makedirs(bdir, exist_ok=True)
    srcs = sources()
    if force:
        for f in os.listdir(bdir):
            if f.endswith(".o"):
                os.remove(os.path.join(bdir, f))
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, bounds), srcs))
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < _newest(objs):
        cmd = [NVCC] + ARCH + ["-shared", "-o", lib] + objs + ["-lcudart_static", "-lrt", "-lpthread", "-ldl"]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, bounds="--bounds" in sys.argv))
