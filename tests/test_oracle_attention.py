"""Pins for the oracle's attention: a naive formula written with Python loops
on tiny inputs, torch's fp64 scaled_dot_product_attention (a library routine,
with an explicit bottom-right causal mask and repeated kv heads for GQA), and
closed-form special cases (rows of P sum to 1, constant V, Q = 0, causal row
0, a single key)."""
import math

import numpy as np
import pytest
import torch

import workloads as wl


def qt_f64_exact(orc, x_f32_bnsd):
    """A bf16 operand (values must be bf16-exact) as an oracle float QT."""
    u = np.ascontiguousarray(x_f32_bnsd, np.float32).view(np.uint32)
    assert (u & 0xFFFF == 0).all()
    return orc.qt_float((u >> 16).astype(np.uint16), "BNSD")


def rand_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16).float().numpy()


def naive(q, k, v, causal, scale):
    """softmax without max subtraction, Python loops (tiny inputs only)."""
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    out = np.zeros((B, Hq, Sq, D))
    lse = np.zeros((B, Hq, Sq))
    for b in range(B):
        for h in range(Hq):
            hk = h // (Hq // Hkv)
            for i in range(Sq):
                ws = []
                for j in range(Sk):
                    if causal and j > i + (Sk - Sq):
                        continue
                    s = sum(float(q[b, h, i, d]) * float(k[b, hk, j, d]) for d in range(D)) * scale
                    ws.append((math.exp(s), j))
                tot = sum(w for w, _ in ws)
                lse[b, h, i] = math.log(tot)
                for d in range(D):
                    out[b, h, i, d] = sum(w * float(v[b, hk, j, d]) for w, j in ws) / tot
    return out, lse


@pytest.mark.parametrize("causal,Sq,Sk,Hq,Hkv", [(False, 5, 7, 2, 2), (True, 6, 6, 4, 2), (True, 3, 8, 2, 1)])
def test_attention_matches_naive_loops(orc, causal, Sq, Sk, Hq, Hkv):
    D = 4
    q = rand_bf16((1, Hq, Sq, D), 1)
    k = rand_bf16((1, Hkv, Sk, D), 2)
    v = rand_bf16((1, Hkv, Sk, D), 3)
    out, lse = orc.attention(qt_f64_exact(orc, q), qt_f64_exact(orc, k), qt_f64_exact(orc, v), causal, 0.0)
    ref, rlse = naive(q, k, v, causal, 1 / math.sqrt(D))
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, rlse, rtol=1e-12, atol=1e-12)


def test_caller_softmax_scale_matches_naive_loops(orc):
    # a positive scale replaces the default 1/sqrt(D) (FlashAttention's softmax_scale)
    D = 4
    q, k, v = rand_bf16((1, 2, 5, D), 4), rand_bf16((1, 1, 9, D), 5), rand_bf16((1, 1, 9, D), 6)
    for scale in (0.37, 2.0):
        out, lse = orc.attention(qt_f64_exact(orc, q), qt_f64_exact(orc, k), qt_f64_exact(orc, v), True, scale)
        ref, rlse = naive(q, k, v, True, scale)
        assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)
        assert np.allclose(lse, rlse, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_attention_matches_torch_sdpa_fp64(orc, causal):
    B, Hq, Hkv, Sq, Sk, D = 2, 8, 2, 37, 53, 64
    q = rand_bf16((B, Hq, Sq, D), 4)
    k = rand_bf16((B, Hkv, Sk, D), 5)
    v = rand_bf16((B, Hkv, Sk, D), 6)
    rows = [0, 5, 17, 36]
    out, _ = orc.attention(qt_f64_exact(orc, q), qt_f64_exact(orc, k), qt_f64_exact(orc, v), causal, 0.0, rows)
    tq, tk, tv = (torch.from_numpy(a).double() for a in (q, k, v))
    tk = tk.repeat_interleave(Hq // Hkv, dim=1)
    tv = tv.repeat_interleave(Hq // Hkv, dim=1)
    mask = None
    if causal:
        i = torch.arange(Sq)[:, None]
        j = torch.arange(Sk)[None, :]
        mask = j <= i + (Sk - Sq)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask)
    assert np.allclose(out, ref[:, :, rows].numpy(), rtol=1e-10, atol=1e-12)


def test_rows_of_p_sum_to_one(orc):
    """With V = the identity (Sk = D keys, key j = e_j), O is the row of P."""
    D = 64
    q = rand_bf16((1, 2, 10, D), 7, 3.0)
    k = rand_bf16((1, 2, D, D), 8, 3.0)
    v = np.tile(np.eye(D, dtype=np.float32), (1, 2, 1, 1))
    for causal in (False, True):
        P, _ = orc.attention(qt_f64_exact(orc, q), qt_f64_exact(orc, k), qt_f64_exact(orc, v), causal, 0.0)
        assert np.allclose(P.sum(-1), 1.0, rtol=0, atol=1e-12)
        assert (P >= 0).all()


def test_constant_v_gives_constant_output(orc):
    q = rand_bf16((1, 2, 9, 64), 9, 4.0)
    k = rand_bf16((1, 2, 50, 64), 10, 4.0)
    v = np.full((1, 2, 50, 64), 1.375, np.float32)
    for causal in (False, True):
        out, _ = orc.attention(qt_f64_exact(orc, q), qt_f64_exact(orc, k), qt_f64_exact(orc, v), causal, 0.0)
        assert np.allclose(out, 1.375, rtol=0, atol=1e-12)


def test_zero_q_gives_mean_of_visible_v(orc):
    Sq = Sk = 12
    q = np.zeros((1, 1, Sq, 64), np.float32)
    k = rand_bf16((1, 1, Sk, 64), 11)
    v = rand_bf16((1, 1, Sk, 64), 12)
    out, lse = orc.attention(qt_f64_exact(orc, q), qt_f64_exact(orc, k), qt_f64_exact(orc, v), True, 0.0)
    for i in range(Sq):
        assert np.allclose(out[0, 0, i], v[0, 0, :i + 1].astype(np.float64).mean(0), rtol=0, atol=1e-12)
        assert abs(lse[0, 0, i] - math.log(i + 1)) < 1e-12
    out, _ = orc.attention(qt_f64_exact(orc, q), qt_f64_exact(orc, k), qt_f64_exact(orc, v), False, 0.0)
    assert np.allclose(out[0, 0], v[0, 0].astype(np.float64).mean(0)[None], rtol=0, atol=1e-12)


def test_causal_row_zero_and_single_key(orc):
    q = rand_bf16((1, 2, 8, 64), 13)
    k = rand_bf16((1, 2, 8, 64), 14)
    v = rand_bf16((1, 2, 8, 64), 15)
    out, _ = orc.attention(qt_f64_exact(orc, q), qt_f64_exact(orc, k), qt_f64_exact(orc, v), True, 0.0)
    assert np.array_equal(out[0, :, 0], v[0, :, 0].astype(np.float64))
    out1, lse1 = orc.attention(qt_f64_exact(orc, q), qt_f64_exact(orc, k[:, :, :1].copy()),
                               qt_f64_exact(orc, v[:, :, :1].copy()), False, 0.0)
    assert np.array_equal(out1, np.broadcast_to(v[:, :, :1].astype(np.float64), out1.shape))


def test_no_visible_key_row(orc):
    """Bottom-right causal alignment with Sq > Sk leaves the first Sq - Sk
    rows without a key: output 0, lse -inf."""
    q = rand_bf16((1, 1, 5, 64), 16)
    k = rand_bf16((1, 1, 3, 64), 17)
    v = rand_bf16((1, 1, 3, 64), 18)
    out, lse = orc.attention(qt_f64_exact(orc, q), qt_f64_exact(orc, k), qt_f64_exact(orc, v), True, 0.0)
    assert not out[0, 0, :2].any() and np.isneginf(lse[0, 0, :2]).all()
    assert np.array_equal(out[0, 0, 2], v[0, 0, 0].astype(np.float64))


def test_quantized_operands_dequantize_per_mode(orc):
    """Attention on quantized operands equals attention on their
    dequantization by hand (code * scale from the format tables)."""
    # B = 2 and H = 3, so that a (b, h) scale index taken as (h, b) lands elsewhere
    x = wl.bf16_bits(wl.normal((2, 3, 64, 64), 19))
    am = orc.calibrate_per_head(x)
    ci, si = orc.quantize_int8_per_head(x, am)
    cf, sf = orc.quantize_fp8_per_token(x)
    cm, em = orc.quantize_mxfp4(x)
    cb, sb = orc.quantize_fp8_block(x, 16)
    qi = orc.QT("int8_per_head", ci, si, 2, 3, 64, 64)
    qf = orc.QT("fp8_per_token", cf, sf, 2, 3, 64, 64)
    qm = orc.QT("mxfp4", cm, em, 2, 3, 64, 64)
    qb = orc.QT("fp8_block", cb, sb, 2, 3, 64, 64, blk=16)
    by_hand = {
        "i": ci.astype(np.float64) * si[None, :, None, None],
        "f": orc.e4m3_decode(cf) * sf[..., None],
        "m": orc.e2m1_decode(np.stack([cm & 15, cm >> 4], -1).reshape(2, 3, 64, 64))
        * np.ldexp(1.0, np.repeat(em.astype(np.int64) - 127, 32, -1)),
        "b": orc.e4m3_decode(cb) * np.repeat(sb, 16, -1)[..., None],
    }
    for key, t in zip("ifmb", (qi, qf, qm, qb)):
        assert np.array_equal(orc.dequant(t), by_hand[key])


def test_mixed_branches_are_attention_on_each_branch_dequantized(orc):
    """fa3_quant details (FA3AttentionDetails): Q, K and V each in its own mode, an unset branch
    left as bf16.  The oracle's attention must equal torch's fp64 SDPA (bottom-right causal mask,
    kv heads repeated for GQA) on each branch dequantized by hand from the format tables."""
    B, Hq, Hkv, S, D = 1, 4, 2, 48, 64
    xq = wl.bf16_bits(wl.normal((B, Hq, S, D), 31))
    xk = wl.bf16_bits(wl.normal((B, Hkv, S, D), 32))
    xv = wl.bf16_bits(wl.normal((B, Hkv, S, D), 33))
    cq, sq = orc.quantize_fp8_per_token(xq)
    ck, sk = orc.quantize_int8_per_head(xk, orc.calibrate_per_head(xk))
    cv, ev = orc.quantize_mxfp4(xv)
    deq = {
        "q": orc.e4m3_decode(cq) * sq[..., None],
        "k": ck.astype(np.float64) * sk[None, :, None, None],
        "v": orc.e2m1_decode(np.stack([cv & 15, cv >> 4], -1).reshape(B, Hkv, S, D))
        * np.ldexp(1.0, np.repeat(ev.astype(np.int64) - 127, 32, -1)),
        "vf": orc.bf16_bits_to_f32(xv).astype(np.float64),
    }
    Q = orc.QT("fp8_per_token", cq, sq, B, Hq, S, D)
    K = orc.QT("int8_per_head", ck, sk, B, Hkv, S, D)
    V = orc.QT("mxfp4", cv, ev, B, Hkv, S, D)
    Vf = orc.qt_float(xv, "BNSD")

    def sdpa(q, k, v, causal):
        k = np.repeat(k, Hq // Hkv, 1)
        v = np.repeat(v, Hq // Hkv, 1)
        mask = None
        if causal:
            mask = torch.ones(S, S, dtype=torch.bool).tril()
        return torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), attn_mask=mask).numpy()

    for causal in (False, True):
        out, _ = orc.attention(Q, K, V, causal, 0.0)
        assert np.allclose(out, sdpa(deq["q"], deq["k"], deq["v"], causal), rtol=1e-12, atol=1e-12)
        out, _ = orc.attention(Q, K, Vf, causal, 0.0)
        assert np.allclose(out, sdpa(deq["q"], deq["k"], deq["vf"], causal), rtol=1e-12, atol=1e-12)
