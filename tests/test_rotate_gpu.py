"""GPU parity for the fused rotate -> FP8 block quantization.

GPU and CPU sum the 128 products of each rotated element in different
orders, so the contract is: every element of the GPU's rotated bf16 tensor
is within half a bf16 ulp plus the fp32 summation bound (127 * 2^-24 *
sum |x_d R_dj| <= 2^-17 * sum |x_d R_dj|) of the oracle's fp64 rotation,
mismatches against the oracle's bf16 rounding are counted, and the codes
and scales are bit-exact against the oracle quantizing the GPU's own
rotated tensor.  With R = I or a signed permutation every sum has one nonzero term,
so the rotated tensor and all codes are exact."""
import numpy as np
import pytest
import torch

import workloads as wl
from _gpu import assert_attention_close, bf16_from_bits, faq_module, head_vmax, np_of, oracle_quantize

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def faq():
    return faq_module()


def ulp_diff(a_bits, b_bits):
    """Distance in bf16 ulps between two arrays of bf16 bit patterns."""
    def key(x):
        x = x.astype(np.int32)
        return np.where(x & 0x8000, -(x & 0x7FFF), x)
    return np.abs(key(a_bits) - key(b_bits))


def shp(B, H, S, layout, D=128):
    return (B, H, S, D) if layout == "BNSD" else (B, S, H, D)


def check_rotated(orc, name, x, R, got, layout, exact=False):
    """The GPU's rotated bf16 tensor (bit patterns) against the oracle's fp64 rotation: within
    half a bf16 ulp plus the fp32 summation bound; returns the fraction differing from the
    oracle's own bf16 rounding (0 required when exact)."""
    xb, Rb = wl.bf16_bits(x), wl.bf16_bits(R)
    exact_f64 = orc.rotate_f64(xb, Rb, layout)
    dist = ulp_diff(got, orc.f64_to_bf16(exact_f64))
    if exact:
        assert dist.max() == 0, name
    absx = np.abs(orc.bf16_bits_to_f32(xb).astype(np.float64))
    absR = np.abs(orc.bf16_bits_to_f32(Rb).astype(np.float64))
    bound = 2.0 ** -17 * (absx @ absR)
    half_ulp = np.ldexp(1.0, np.frexp(np.abs(exact_f64))[1] - 9)
    err = np.abs(orc.bf16_bits_to_f32(got).astype(np.float64) - exact_f64)
    assert (err <= bound + half_ulp + 1e-300).all(), f"{name}: rotation outside the fp32 summation bound"
    return float((dist > 0).mean())


def check_rotate(faq, orc, q, k, v, Rq, Rk, layout, q_blk, kv_blk, exact=False):
    Q, K, V, dq, dk = faq.rotate_quantize(q.cuda(), k.cuda(), v.cuda(), Rq.cuda(), Rk.cuda(), layout,
                                          q_blk, kv_blk, debug=True)
    faq.check_device_status()
    stats = {}
    for name, x, R, d, out, blk in (("q", q, Rq, dq, Q, q_blk), ("k", k, Rk, dk, K, kv_blk)):
        got = np_of(d)
        stats[name] = check_rotated(orc, name, x, R, got, layout, exact)
        codes, scales = orc.quantize_fp8_block(got, blk, layout)
        assert np.array_equal(np_of(out.scales), scales), name
        assert np.array_equal(np_of(out.codes), codes), name
    codes, scales = orc.quantize_fp8_block(wl.bf16_bits(v), kv_blk, layout)
    assert np.array_equal(np_of(V.scales), scales)
    assert np.array_equal(np_of(V.codes), codes)
    return stats, (Q, K, V)


@pytest.mark.parametrize("layout,S,q_blk,kv_blk", [("BSND", 300, 128, 256), ("BNSD", 513, 128, 256),
                                                  ("BSND", 100, 64, 32), ("BNSD", 256, 256, 256)])
def test_rotate_block_quant(faq, orc, layout, S, q_blk, kv_blk):
    q = wl.normal(shp(2, 3, S, layout), 1)
    k = wl.normal(shp(2, 3, S, layout), 2)
    v = wl.normal(shp(2, 3, S, layout), 3)
    R = wl.rotation(128, 5)
    stats, _ = check_rotate(faq, orc, q, k, v, R, R, layout, q_blk, kv_blk)
    assert stats["q"] < 1e-2 and stats["k"] < 1e-2


def test_rotate_many_items_per_cta(faq, orc):
    """More 256-token chunks than SMs: each persistent CTA walks items of several operands
    (Q, then K, then V), so the resident rotation is swapped mid-stream; distinct R_q and R_k
    make a stale rotation show."""
    B, H, S = 2, 8, 5000  # 20 chunks per (b, h): 960 items
    q = wl.normal(shp(B, H, S, "BSND"), 31)
    k = wl.normal(shp(B, H, S, "BSND"), 32)
    v = wl.normal(shp(B, H, S, "BSND"), 33)
    Rq = wl.rotation(128, 34)
    Rk = (wl.normal((128, 128), 35).float() * 0.1).to(torch.bfloat16)
    stats, _ = check_rotate(faq, orc, q, k, v, Rq, Rk, "BSND", 128, 256)
    assert stats["q"] < 1e-2


def test_rotate_key_only_through_abi(faq, orc):
    """Only K passed through the C ABI (Q and V null): K's rotation is the first one resident."""
    import ctypes
    from quantized_attention_amax_b200 import _native as N, api
    k = wl.normal((1, 700, 3, 128), 41).cuda()
    Rk = (wl.normal((128, 128), 42).float() * 0.1).to(torch.bfloat16).cuda()
    K = api.empty_qtensor(1, 3, 700, 128, "fp8_block", "BSND", 256, k.device)
    tk, ck = api._tensor(k, "BSND"), K.c()
    dk = torch.empty_like(k)
    st = N.lib().fa_rotate_quantize(None, ctypes.byref(tk), None, None, Rk.data_ptr(), 128, 256, None,
                                    ctypes.byref(ck), None, None, dk.data_ptr(), api._stream())
    assert st == 0
    faq.check_device_status()
    got = np_of(dk)
    check_rotated(orc, "k", k.cpu(), Rk.cpu(), got, "BSND")
    codes, scales = orc.quantize_fp8_block(got, 256, "BSND")
    assert np.array_equal(np_of(K.scales), scales)
    assert np.array_equal(np_of(K.codes), codes)


def test_rotate_general_matrix_catches_transpose(faq, orc):
    """A non-symmetric R and distinct R_q, R_k: x R (not R x, not x R^T)."""
    q = wl.normal((1, 200, 2, 128), 11)
    k = wl.normal((1, 200, 2, 128), 12)
    v = wl.normal((1, 200, 2, 128), 13)
    Rq = (wl.normal((128, 128), 14).float() * 0.1).to(torch.bfloat16)
    Rk = (wl.normal((128, 128), 15).float() * 0.1).to(torch.bfloat16)
    check_rotate(faq, orc, q, k, v, Rq, Rk, "BSND", 128, 256)


def test_rotate_identity_and_signed_permutation_exact(faq, orc):
    q = wl.normal((1, 300, 2, 128), 21)
    k = wl.normal((1, 300, 2, 128), 22)
    v = wl.normal((1, 300, 2, 128), 23)
    eye = torch.eye(128).to(torch.bfloat16)
    _, (Q, K, V) = check_rotate(faq, orc, q, k, v, eye, eye, "BSND", 128, 256, exact=True)
    cq, sq = orc.quantize_fp8_block(wl.bf16_bits(q), 128, "BSND")
    assert np.array_equal(np_of(Q.codes), cq) and np.array_equal(np_of(Q.scales), sq)
    rng = np.random.default_rng(3)
    perm = rng.permutation(128)
    sign = rng.choice([-1.0, 1.0], 128)
    P = np.zeros((128, 128), np.float32)
    P[perm, np.arange(128)] = sign
    Pt = torch.from_numpy(P).to(torch.bfloat16)
    _, (Q2, K2, _) = check_rotate(faq, orc, q, k, v, Pt, Pt, "BSND", 128, 256, exact=True)
    ck, sk = orc.quantize_fp8_block(wl.bf16_bits(k), 256, "BSND")
    flip = np.where(sign < 0, 0x80, 0).astype(np.uint8)
    assert np.array_equal(np_of(K2.codes), ck[..., perm] ^ flip)
    assert np.array_equal(np_of(K2.scales), sk)


def test_full_size_rotate_workload(faq, orc):
    """The video-DiT workload at full size (B=1, H=40, S=32768, BSND): the
    rotation and codes as above, then attention on sampled query rows vs the
    oracle's own rotate -> block-quant -> attention pipeline."""
    w = wl.WORKLOADS["rot_fp8_block"]
    inp = wl.make_inputs(w)
    stats, (Q, K, V) = check_rotate(faq, orc, inp["q"], inp["k"], inp["v"], inp["R"], inp["R"], w.layout,
                                    w.q_block, w.kv_block)
    assert stats["q"] < 1e-2 and stats["k"] < 1e-2
    out = faq.attention(Q, K, V, causal=False)
    faq.check_device_status()
    Rb = wl.bf16_bits(inp["R"])
    oq = oracle_quantize(orc, "fp8_block", orc.rotate(wl.bf16_bits(inp["q"]), Rb, w.layout), w.layout, w.q_block)
    ok_ = oracle_quantize(orc, "fp8_block", orc.rotate(wl.bf16_bits(inp["k"]), Rb, w.layout), w.layout, w.kv_block)
    ov = oracle_quantize(orc, "fp8_block", wl.bf16_bits(inp["v"]), w.layout, w.kv_block)
    rng = np.random.default_rng(1)
    rows = sorted(set([0, 127, 128, 255, 256, w.Sq - 1] + list(rng.choice(w.Sq, 40, False))))
    ref, _ = orc.attention(oq, ok_, ov, False, 0.0, rows)
    got = np.ascontiguousarray(np_of(out.float()).transpose(0, 2, 1, 3))[:, :, rows, :]
    assert_attention_close(got, ref, head_vmax(orc, ov, w.Hq), "rot_fp8_block")
