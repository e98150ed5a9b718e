"""Random arguments through every C-ABI entry point: the host-side checks never crash.

Shapes take edge values (negative, zero, odd, past 2^31 when multiplied), modes and layouts
go out of range, and pointers are NULL, misaligned or made up.  Every call must return a known
fa_status (or a size) instead of crashing the process.  A made-up pointer that passes the
checks would reach a kernel launch, so the calls run in a child process that can see no GPU at
all (CUDA_VISIBLE_DEVICES is empty): any launch fails with FA_ERR_CUDA and no device memory is
touched.
"""
import ctypes
import os
import random
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
STATUSES = set(range(8))  # FA_OK .. FA_ERR_WORKSPACE
VALS = [-2 ** 31, -5, -1, 0, 1, 2, 3, 7, 16, 31, 32, 33, 63, 64, 100, 127, 128, 129, 255, 256, 4096, 32768,
        65535, 65536, 2 ** 20, 2 ** 30, 2 ** 31 - 1]


def child(seed: int, iters: int) -> None:
    assert os.environ.get("CUDA_VISIBLE_DEVICES") == ""
    sys.path.insert(0, ROOT)
    from quantized_attention_amax_b200 import _native as N
    L = N.lib()
    rnd = random.Random(seed)

    def rint():
        return rnd.choice(VALS)

    def rptr():
        return rnd.choice([None, 0x100000, 0x100008, 0x100004, 0x7F0000000000])

    def qt():
        t = N.FaQTensor()
        t.codes, t.scales = rptr(), rptr()
        t.mode = rnd.choice([-1, 0, 1, 2, 3, 4, 5, 6, 7, 8])
        t.B, t.H, t.S = rint(), rint(), rint()
        t.D = rnd.choice([0, 32, 64, 96, 128, 256, rint()])
        t.layout = rnd.choice([-1, 0, 1, 2])
        t.block_tokens = rint()
        return t

    def ft():
        t = N.FaTensor()
        t.data = rptr()
        t.B, t.H, t.S = rint(), rint(), rint()
        t.D = rnd.choice([0, 64, 128, rint()])
        t.layout = rnd.choice([0, 1, 5])
        return t

    R = ctypes.byref
    for _ in range(iters):
        q, k, v = qt(), qt(), qt()
        if rnd.random() < 0.5:  # consistent operands reach the deeper checks
            k.mode = v.mode = q.mode
            k.D = v.D = q.D
            k.B = v.B = q.B
            k.layout = v.layout = q.layout
            v.H, v.S = k.H, k.S
        f = rnd.randrange(7)
        if f == 0:
            L.fa_attention_workspace_size(R(q), R(k), rint())
            continue
        if f == 1:
            L.fa_attention_workspace_size_qkv(R(q), R(k), R(v), rint())
            continue
        if f == 6:
            L.fa_decode_append_workspace_size(R(ft()), R(k), rint(), rint())
            continue
        if f == 2:
            st = L.fa_attention_quant(R(q), R(k), R(v), rnd.randrange(2), 0.0, rptr(), rptr(), rint() % 64, rptr(),
                                      rint() & 0xFFFFFFFF, None)
        elif f == 3:
            st = L.fa_attention_decode_noalloc(R(q), R(k), R(v), 0.0, rptr(), rptr(), rint() % 64, None)
        elif f == 4:
            st = L.fa_quantize(R(ft()), R(ft()), R(ft()), rnd.randrange(-1, 9), rptr(), rptr(), rptr(), R(q), R(k),
                               R(v), None)
        else:
            st = L.fa_rotate_quantize(R(ft()), R(ft()), R(ft()), rptr(), rptr(), rint(), rint(), R(q), R(k), R(v),
                                      rptr(), rptr(), None)
        assert st in STATUSES, st
    print("fuzz ok")


@pytest.mark.parametrize("seed", [1, 2])
def test_random_arguments_never_crash_the_host_checks(seed):
    from quantized_attention_amax_b200 import build
    build.build()
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.abspath(__file__), str(seed), "4000"], capture_output=True,
                       text=True, env=env, timeout=600)
    assert r.returncode == 0 and "fuzz ok" in r.stdout, (r.returncode, r.stdout[-2000:], r.stderr[-2000:])


if __name__ == "__main__":
    child(int(sys.argv[1]), int(sys.argv[2]))
