"""The allocation-free decode entry point (fa_attention_decode_noalloc).

It is for callers that cannot allocate device memory where they run decode
(a serving loop that must not synchronise the device, or C/C++ host code
without a device allocator): its split-KV partials live in a fixed buffer
inside libfaq.so instead of a caller workspace.  These tests call it through
the C ABI and compare it with the existing entry point, fa_attention_quant,
on two calls in a row, within the attention tolerance the other tests use.
This file is collected last on purpose (test_zz_*)."""
import ctypes

import numpy as np
import pytest
import torch

import workloads as wl
from _gpu import ATOL_MAX, ATOL_MEAN, faq_module, np_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def faq():
    return faq_module()


def setup(faq, B=2, Hq=8, Hkv=2, Sk=5000, seed=77):
    q = wl.normal((B, Hq, 1, 128), seed).cuda()
    k = wl.normal((B, Hkv, Sk, 128), seed + 1).cuda()
    v = wl.normal((B, Hkv, Sk, 128), seed + 2).cuda()
    amax = [faq.calibrate_per_head(wl.normal(t.shape, seed + 10 + i).cuda()) for i, t in enumerate((q, k, v))]
    return faq.quantize(q, k, v, "int8_per_head", amax=amax)


def noalloc(faq, Q, K, V, splits=0):
    from quantized_attention_amax_b200 import _native as N
    out = torch.empty((Q.B, Q.H, 1, Q.D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((Q.B, Q.H, 1), dtype=torch.float32, device="cuda")
    cq, ck, cv = Q.c(), K.c(), V.c()
    st = N.lib().fa_attention_decode_noalloc(ctypes.byref(cq), ctypes.byref(ck), ctypes.byref(cv), 0.0,
                                             out.data_ptr(), lse.data_ptr(), splits,
                                             torch.cuda.current_stream().cuda_stream)
    return st, out, lse


def close(a, b, M):
    err = np.abs(np_of(a.float()).astype(np.float64) - np_of(b.float()))
    return err.max() <= ATOL_MAX * M and err.mean() <= ATOL_MEAN * M


def test_noalloc_matches_decode_twice(faq):
    Q, K, V = setup(faq)
    ref, ref_lse = faq.attention(Q, K, V, return_lse=True)
    faq.check_device_status()
    M = float(np.abs(np_of(V.codes).astype(np.float64)).max() * np_of(V.scales).max())
    for _ in range(2):
        st, out, lse = noalloc(faq, Q, K, V)
        assert st == 0
        faq.check_device_status()
        assert close(out, ref, M)
        assert np.abs(np_of(lse) - np_of(ref_lse)).max() < 1e-3 * max(1.0, np.abs(np_of(ref_lse)).max())
    # same split count -> same kernels, same result
    st, out2, _ = noalloc(faq, Q, K, V, splits=3)
    ref3 = faq.attention(Q, K, V, num_splits=3)
    faq.check_device_status()
    assert st == 0 and close(out2, ref3, M)


def test_noalloc_rejects_oversized_partials(faq):
    Q, K, V = setup(faq, B=16, Hq=32, Hkv=8, Sk=300)
    from quantized_attention_amax_b200 import _native as N
    # 16 * 32 * splits * 130 * 4 bytes > 16 MiB once splits > 62
    st, _, _ = noalloc(faq, Q, K, V, splits=200)
    assert st == 7  # FA_ERR_WORKSPACE, rejected before any launch
    st, out, _ = noalloc(faq, Q, K, V)  # automatic split count fits
    assert st == 0
    faq.check_device_status()
