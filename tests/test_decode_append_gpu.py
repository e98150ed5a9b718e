"""GPU parity for fa_decode_append: one decode step that quantizes the new token's K / V into an
INT8 per-head cache at `pos` and attends over the first pos + 1 cached tokens, with the query
quantized in the decode kernel.  The cache afterwards must hold exactly the oracle's codes of
the whole history (earlier rows from fa_quantize, row pos from the append) and the output must
match the oracle's attention over the prefix."""
import numpy as np
import pytest
import torch

import workloads as wl
from _gpu import assert_attention_close, faq_module, head_vmax, np_of, oracle_quantize

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def faq():
    return faq_module()


def tok(t, layout, lo, hi):
    """Tokens [lo, hi) of a [B, H, S, D] / [B, S, H, D] tensor."""
    return (t[:, :, lo:hi] if layout == "BNSD" else t[:, lo:hi]).contiguous()


@pytest.mark.parametrize("layout,B,Hq,Hkv,cap,pos,splits", [
    ("BNSD", 2, 8, 2, 700, 0, 0), ("BNSD", 2, 8, 2, 700, 128, 0), ("BNSD", 2, 8, 2, 700, 699, 0),
    ("BSND", 1, 4, 4, 1000, 517, 3), ("BNSD", 1, 16, 1, 300, 255, 1), ("BSND", 3, 8, 1, 257, 200, 2)])
def test_decode_append_matches_oracle(faq, orc, layout, B, Hq, Hkv, cap, pos, splits):
    D = 128
    shp = lambda H, S: (B, H, S, D) if layout == "BNSD" else (B, S, H, D)
    seed = 7 * pos + Hq + cap
    hist = {n: wl.normal(shp(Hkv, cap), seed + i) for i, n in enumerate("kv")}
    q = wl.normal(shp(Hq, 1), seed + 2)
    cal = {"q": wl.normal(shp(Hq, 1), seed + 10), "k": wl.normal(shp(Hkv, cap), seed + 11),
           "v": wl.normal(shp(Hkv, cap), seed + 12)}
    amax = {n: orc.calibrate_per_head(wl.bf16_bits(cal[n]), layout) for n in "qkv"}
    am = [torch.from_numpy(amax[n]).cuda() for n in "qkv"]
    # the cache: every row quantized, then row pos and the scales overwritten with junk
    _, Kc, Vc = faq.quantize(None, hist["k"].cuda(), hist["v"].cuda(), "int8_per_head", layout, amax=[None, am[1], am[2]])
    for c in (Kc, Vc):
        (c.codes[:, :, pos] if layout == "BNSD" else c.codes[:, pos]).fill_(77)
        c.scales.fill_(123.0)
    out, lse = faq.decode_append(q.cuda(), tok(hist["k"], layout, pos, pos + 1).cuda(),
                                 tok(hist["v"], layout, pos, pos + 1).cuda(), am, Kc, Vc, pos,
                                 num_splits=splits, return_lse=True)
    faq.check_device_status()
    for n, c in zip("kv", (Kc, Vc)):
        codes, scales = orc.quantize_int8_per_head(wl.bf16_bits(hist[n]), amax[n], layout)
        assert np.array_equal(np_of(c.codes), codes)
        assert np.array_equal(np_of(c.scales), scales)
    oq = oracle_quantize(orc, "int8_per_head", wl.bf16_bits(q), layout, 0, amax["q"])
    ok_, ov = (oracle_quantize(orc, "int8_per_head", wl.bf16_bits(tok(hist[n], layout, 0, pos + 1)), layout, 0, amax[n])
               for n in "kv")
    ref, ref_lse = orc.attention(oq, ok_, ov, False, 0.0)
    got = np_of(out.float())
    if layout == "BSND":
        got = np.ascontiguousarray(got.transpose(0, 2, 1, 3))
    assert_attention_close(got, ref, head_vmax(orc, ov, Hq), f"decode_append pos={pos}")
    assert np.abs(np_of(lse) - ref_lse).max() < 2e-3 * max(1.0, np.abs(ref_lse).max())


def test_decode_append_steps_build_the_cache(faq, orc):
    """Several steps in a row: each appends its token; after them the cache equals the
    quantization of the whole sequence and the last output matches the oracle."""
    B, Hq, Hkv, cap, D = 1, 4, 2, 160, 128
    hist = {n: wl.normal((B, Hkv, cap, D), 90 + i) for i, n in enumerate("kv")}
    amax = {n: orc.calibrate_per_head(wl.bf16_bits(hist[n]), "BNSD") for n in "kv"}
    amax["q"] = np.full(Hq, 4.0, np.float32)
    am = [torch.from_numpy(amax[n]).cuda() for n in "qkv"]
    start = 100
    _, Kc, Vc = faq.quantize(None, hist["k"].cuda(), hist["v"].cuda(), "int8_per_head", "BNSD", amax=[None, am[1], am[2]])
    Kc.codes[:, :, start:].zero_()
    Vc.codes[:, :, start:].zero_()
    for pos in range(start, cap):
        q = wl.normal((B, Hq, 1, D), 200 + pos)
        out = faq.decode_append(q.cuda(), hist["k"][:, :, pos:pos + 1].contiguous().cuda(),
                                hist["v"][:, :, pos:pos + 1].contiguous().cuda(), am, Kc, Vc, pos)
    faq.check_device_status()
    for n, c in zip("kv", (Kc, Vc)):
        codes, _ = orc.quantize_int8_per_head(wl.bf16_bits(hist[n]), amax[n], "BNSD")
        assert np.array_equal(np_of(c.codes), codes)
    oq = oracle_quantize(orc, "int8_per_head", wl.bf16_bits(q), "BNSD", 0, amax["q"])
    ok_, ov = (oracle_quantize(orc, "int8_per_head", wl.bf16_bits(hist[n]), "BNSD", 0, amax[n]) for n in "kv")
    ref, _ = orc.attention(oq, ok_, ov, False, 0.0)
    assert_attention_close(np_of(out.float()), ref, head_vmax(orc, ov, Hq), "decode_append steps")
