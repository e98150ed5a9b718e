"""GPU parity for the Hadamard rotation path (fa_rotate_quantize_hadamard): R =
bf16(H_D diag(sigma) / sqrt(D)) applied by a fast Walsh-Hadamard transform.  The contract is
the general rotation's: every element of the GPU's rotated bf16 tensor within half a bf16 ulp
plus the fp32 summation bound of the oracle's fp64 rotation x R (R materialized from the same
signs), and the codes and scales bit-exact against the oracle quantizing the GPU's own rotated
tensor.  V is block-quantized without rotation, bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import workloads as wl
from _gpu import assert_attention_close, faq_module, head_vmax, np_of, oracle_quantize
from test_rotate_gpu import check_rotated, shp

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def faq():
    return faq_module()


def hadamard_R(D, signs):
    """bf16 [D, D] = bf16(H_D diag(signs) / sqrt(D)) (the matrix the fast path stands for)."""
    Hm = torch.ones(1, 1, dtype=torch.float64)
    while Hm.shape[0] < D:
        Hm = torch.cat([torch.cat([Hm, Hm], 1), torch.cat([Hm, -Hm], 1)], 0)
    s = torch.tensor(signs if signs is not None else [1] * D, dtype=torch.float64)
    return (Hm * s[None, :] / D ** 0.5).to(torch.bfloat16)


def check_hadamard(faq, orc, q, k, v, sq, sk, layout, q_blk, kv_blk):
    D = q.shape[-1]
    Q, K, V, dq, dk = faq.rotate_quantize_hadamard(q.cuda(), k.cuda(), v.cuda(), sq, sk, layout, q_blk, kv_blk,
                                                   debug=True)
    faq.check_device_status()
    stats = {}
    for name, x, sg, d, out, blk in (("q", q, sq, dq, Q, q_blk), ("k", k, sk, dk, K, kv_blk)):
        got = np_of(d)
        stats[name] = check_rotated(orc, name, x, hadamard_R(D, sg), got, layout)
        codes, scales = orc.quantize_fp8_block(got, blk, layout)
        assert np.array_equal(np_of(out.scales), scales), name
        assert np.array_equal(np_of(out.codes), codes), name
    codes, scales = orc.quantize_fp8_block(wl.bf16_bits(v), kv_blk, layout)
    assert np.array_equal(np_of(V.scales), scales)
    assert np.array_equal(np_of(V.codes), codes)
    return stats, (Q, K, V)


@pytest.mark.parametrize("layout,D,S,q_blk,kv_blk", [
    ("BSND", 128, 300, 128, 256),   # ragged last blocks
    ("BNSD", 128, 513, 128, 256),
    ("BSND", 64, 100, 64, 32),
    ("BNSD", 128, 256, 256, 256),
    ("BNSD", 128, 700, 100, 300),   # blocks that do not divide the tile; 300 rows exceed the kept-row buffer
    ("BSND", 64, 1000, 1000, 700),  # 64-dim rows, long blocks
])
def test_hadamard_block_quant(faq, orc, layout, D, S, q_blk, kv_blk):
    q = wl.normal(shp(2, 3, S, layout, D), 1)
    k = wl.normal(shp(2, 3, S, layout, D), 2)
    v = wl.normal(shp(2, 3, S, layout, D), 3)
    sq = wl.rotation_signs(D, 5)
    sk = wl.rotation_signs(D, 6)
    stats, _ = check_hadamard(faq, orc, q, k, v, sq, sk, layout, q_blk, kv_blk)
    assert stats["q"] < 1e-2 and stats["k"] < 1e-2


def test_hadamard_without_signs_and_outliers(faq, orc):
    """All signs +1 (NULL sign words), K with x20 outlier channels and a zero block."""
    q = wl.normal((1, 2, 384, 128), 7)
    k = wl.normal_k_outliers((1, 2, 384, 128), "BNSD", 8)
    v = wl.normal((1, 2, 384, 128), 9)
    k[:, :, 128:256] = 0
    stats, (_, K, _) = check_hadamard(faq, orc, q, k, v, None, None, "BNSD", 128, 128)
    assert np_of(K.scales)[0, 0, 1] == 0.0 and (np_of(K.codes)[0, 0, 128:256] == 0).all()


def test_hadamard_matches_general_rotation(faq, orc):
    """The fast path and fa_rotate_quantize with the materialized R agree on almost every rotated
    element (they differ only in the order of the fp32 sums), and wherever a block's rotated
    values agree, its scale and codes agree."""
    q = wl.normal((1, 600, 4, 128), 21)
    k = wl.normal((1, 600, 4, 128), 22)
    v = wl.normal((1, 600, 4, 128), 23)
    sg = wl.rotation_signs(128, 24)
    R = hadamard_R(128, sg).cuda()
    Qh, Kh, Vh, dqh, dkh = faq.rotate_quantize_hadamard(q.cuda(), k.cuda(), v.cuda(), sg, sg, "BSND", 128, 256,
                                                        debug=True)
    Qg, Kg, Vg, dqg, dkg = faq.rotate_quantize(q.cuda(), k.cuda(), v.cuda(), R, R, "BSND", 128, 256, debug=True)
    faq.check_device_status()
    for a, b in ((dqh, dqg), (dkh, dkg)):
        assert (np_of(a) != np_of(b)).mean() < 1e-2
    assert np.array_equal(np_of(Vh.codes), np_of(Vg.codes)) and np.array_equal(np_of(Vh.scales), np_of(Vg.scales))


def test_full_size_hadamard_workload(faq, orc):
    """The video-DiT workload at full size through the fast path (its R is Hadamard x signs):
    rotation and codes as above, then attention on sampled rows vs the oracle's pipeline."""
    w = wl.WORKLOADS["rot_fp8_block"]
    inp = wl.make_inputs(w)
    sg = wl.rotation_signs(w.D, w.seed)
    assert torch.equal(hadamard_R(w.D, sg), inp["R"])
    stats, (Q, K, V) = check_hadamard(faq, orc, inp["q"], inp["k"], inp["v"], sg, sg, w.layout, w.q_block,
                                      w.kv_block)
    assert stats["q"] < 1e-2 and stats["k"] < 1e-2
    out = faq.attention(Q, K, V, causal=False)
    faq.check_device_status()
    Rb = wl.bf16_bits(inp["R"])
    oq = oracle_quantize(orc, "fp8_block", orc.rotate(wl.bf16_bits(inp["q"]), Rb, w.layout), w.layout, w.q_block)
    ok_ = oracle_quantize(orc, "fp8_block", orc.rotate(wl.bf16_bits(inp["k"]), Rb, w.layout), w.layout, w.kv_block)
    ov = oracle_quantize(orc, "fp8_block", wl.bf16_bits(inp["v"]), w.layout, w.kv_block)
    rng = np.random.default_rng(2)
    rows = sorted(set([0, 127, 128, 255, 256, w.Sq - 1] + list(rng.choice(w.Sq, 40, False))))
    ref, _ = orc.attention(oq, ok_, ov, False, 0.0, rows)
    got = np.ascontiguousarray(np_of(out.float()).transpose(0, 2, 1, 3))[:, :, rows, :]
    assert_attention_close(got, ref, head_vmax(orc, ov, w.Hq), "rot_fp8_block (Hadamard path)")
