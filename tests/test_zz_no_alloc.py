"""The allocation-free decode entry point (fa_attention_decode_noalloc).

It serves callers that cannot allocate device memory at the point where they
run decode: a serving loop that must never synchronise the device (cudaMalloc
and cudaFree can), or C/C++ host code that links libfaq.so and has no device
allocator.  Its split-KV partials live in a fixed buffer inside the library
instead of a caller workspace.

These tests call it through the C ABI and check its output against the oracle's
exact fp64 attention (per-head M_h, the tolerance every attention test uses)
and against the existing entry point, fa_attention_quant, on two calls in a row;
they also reach the code that lowers the automatic split count until the
partials fit the buffer, and check that a call leaves the device's free memory
unchanged.  This file is collected last on purpose (test_zz_*)."""
import ctypes

import numpy as np
import pytest
import torch

import workloads as wl
from _gpu import assert_attention_close, faq_module, head_vmax, np_of, oracle_quantize

pytestmark = pytest.mark.gpu

FA_OK, FA_ERR_WORKSPACE = 0, 7


@pytest.fixture(scope="module")
def faq():
    return faq_module()


def setup(faq, orc, B=2, Hq=8, Hkv=2, Sk=5000, seed=77):
    """Seeded bf16 Q/K/V and calibration batches -> the GPU's INT8 per-head operands and the
    oracle's own quantization of the same bf16 inputs."""
    q = wl.normal((B, Hq, 1, 128), seed)
    k = wl.normal((B, Hkv, Sk, 128), seed + 1)
    v = wl.normal((B, Hkv, Sk, 128), seed + 2)
    amax = {n: orc.calibrate_per_head(wl.bf16_bits(wl.normal(t.shape, seed + 10 + i)))
            for i, (n, t) in enumerate(zip("qkv", (q, k, v)))}
    oq = {n: oracle_quantize(orc, "int8_per_head", wl.bf16_bits(t), "BNSD", 0, amax[n])
          for n, t in zip("qkv", (q, k, v))}
    am = [torch.from_numpy(amax[n]).cuda() for n in "qkv"]
    Q, K, V = faq.quantize(q.cuda(), k.cuda(), v.cuda(), "int8_per_head", amax=am)
    return (Q, K, V), oq


def noalloc(Q, K, V, splits=0, out=None, lse=None):
    from quantized_attention_amax_b200 import _native as N
    if out is None:
        out = torch.empty((Q.B, Q.H, 1, Q.D), dtype=torch.bfloat16, device="cuda")
    if lse is None:
        lse = torch.empty((Q.B, Q.H, 1), dtype=torch.float32, device="cuda")
    cq, ck, cv = Q.c(), K.c(), V.c()
    st = N.lib().fa_attention_decode_noalloc(ctypes.byref(cq), ctypes.byref(ck), ctypes.byref(cv), 0.0,
                                             out.data_ptr(), lse.data_ptr(), splits,
                                             torch.cuda.current_stream().cuda_stream)
    return st, out, lse


def test_noalloc_matches_oracle_and_decode_twice(faq, orc):
    (Q, K, V), oq = setup(faq, orc)
    ref, ref_lse = orc.attention(oq["q"], oq["k"], oq["v"], False, 0.0)
    M = head_vmax(orc, oq["v"], Q.H)
    lib_out, lib_lse = faq.attention(Q, K, V, return_lse=True)
    faq.check_device_status()
    for call in range(2):
        st, out, lse = noalloc(Q, K, V)
        assert st == FA_OK
        faq.check_device_status()
        got = np_of(out.float())
        assert_attention_close(got, ref, M, f"noalloc call {call} vs oracle")
        assert_attention_close(got, np_of(lib_out.float()).astype(np.float64), M,
                               f"noalloc call {call} vs fa_attention_quant")
        assert np.abs(np_of(lse) - ref_lse).max() < 2e-3 * max(1.0, np.abs(ref_lse).max())
        assert np.abs(np_of(lse) - np_of(lib_lse)).max() < 1e-3 * max(1.0, np.abs(ref_lse).max())
    # a caller's split count: the same kernels as fa_attention_quant with that count
    st, out3, _ = noalloc(Q, K, V, splits=3)
    lib3 = faq.attention(Q, K, V, num_splits=3)
    faq.check_device_status()
    assert st == FA_OK
    assert_attention_close(np_of(out3.float()), ref, M, "noalloc splits=3 vs oracle")
    assert np.array_equal(np_of(out3), np_of(lib3))


def test_noalloc_rejects_oversized_partials(faq, orc):
    (Q, K, V), _ = setup(faq, orc, B=16, Hq=32, Hkv=8, Sk=300)
    # 16 * 32 * splits * 130 * 4 bytes > 16 MiB once splits > 62: rejected before any launch
    st, _, _ = noalloc(Q, K, V, splits=200)
    assert st == FA_ERR_WORKSPACE
    st, _, _ = noalloc(Q, K, V)  # the automatic split count fits
    assert st == FA_OK
    faq.check_device_status()


def test_noalloc_lowers_automatic_splits_and_allocates_nothing(faq, orc):
    """B * Hq = 16384 query rows over 4096 keys: the automatic split count (2) would need
    16.25 MiB of partials, so the call lowers it to one split; its output then equals
    fa_attention_quant's with one split, and matches the oracle on sampled batches."""
    B, Hq, Hkv, Sk, D = 128, 128, 8, 4096, 128
    g = torch.Generator(device="cuda")
    g.manual_seed(2024)
    mk = lambda *s: torch.randn(s, generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)
    q, k, v = mk(B, Hq, 1, D), mk(B, Hkv, Sk, D), mk(B, Hkv, Sk, D)
    am = [faq.calibrate_per_head(mk(*t.shape)) for t in (q, k, v)]
    Q, K, V = faq.quantize(q, k, v, "int8_per_head", amax=am)
    del k, v
    auto = faq.attention_workspace_size(Q, K) // (B * Hq * (D + 2) * 4)
    assert auto * B * Hq * (D + 2) * 4 > (16 << 20), "the shape must overflow the buffer at the automatic count"
    out = torch.empty((B, Hq, 1, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq, 1), dtype=torch.float32, device="cuda")
    st, out, lse = noalloc(Q, K, V, out=out, lse=lse)
    assert st == FA_OK
    faq.check_device_status()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    st, out, lse = noalloc(Q, K, V, out=out, lse=lse)  # second call, same buffers
    assert st == FA_OK
    faq.check_device_status()
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0, "the call changed the device's free memory"
    ref1 = faq.attention(Q, K, V, num_splits=1)
    faq.check_device_status()
    assert np.array_equal(np_of(out), np_of(ref1))
    # oracle on two batches (first and last), from the GPU's codes
    for b in (0, B - 1):
        sub = lambda t: orc.QT(t.mode, np.ascontiguousarray(np_of(t.codes)[b:b + 1]), np_of(t.scales), 1, t.H, t.S,
                               t.D, "BNSD", 0)
        qo, ko, vo = sub(Q), sub(K), sub(V)
        ref, _ = orc.attention(qo, ko, vo, False, 0.0)
        assert_attention_close(np_of(out.float())[b:b + 1], ref, head_vmax(orc, vo, Hq), f"batch {b}")
