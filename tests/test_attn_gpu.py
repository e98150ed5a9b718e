"""GPU parity for prefill attention on quantized operands: the CUDA path vs
the oracle's exact fp64 attention on the oracle's own quantization of the
same seeded inputs (the codes agree bit for bit, so both see the same
operands), within max <= 2e-2 M_h and mean <= 2e-3 M_h."""
import numpy as np
import pytest
import torch

import workloads as wl
from _gpu import assert_attention_close, faq_module, head_vmax, np_of, oracle_quantize

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def faq():
    return faq_module()


def shp(B, H, S, D, layout):
    return (B, H, S, D) if layout == "BNSD" else (B, S, H, D)


def to_bnsd(a, layout):
    return a if layout == "BNSD" else np.ascontiguousarray(a.transpose(0, 2, 1, 3))


def run_case(faq, orc, mode, layout, D, B, Hq, Hkv, Sq, Sk, causal, seed, q_blk=128, kv_blk=256, rows=None,
             dist=None, lse=True):
    if dist is None:
        dist = "t4" if mode in ("mxfp4", "mxfp8") else "normal"
    gen = wl.student_t4 if dist == "t4" else wl.normal
    q = gen(shp(B, Hq, Sq, D, layout), seed)
    k = gen(shp(B, Hkv, Sk, D, layout), seed + 1)
    v = gen(shp(B, Hkv, Sk, D, layout), seed + 2)
    bits = {n: wl.bf16_bits(t) for n, t in zip("qkv", (q, k, v))}
    amax = {}
    if mode in ("int8_per_head", "fp8_per_head"):
        for n, t in zip("qkv", (q, k, v)):
            cal = gen(t.shape, seed + 50 + "qkv".index(n))
            amax[n] = orc.calibrate_per_head(wl.bf16_bits(cal), layout)
    blks = {"q": q_blk, "k": kv_blk, "v": kv_blk}
    oq = {n: oracle_quantize(orc, mode, bits[n], layout, blks[n] if mode == "fp8_block" else 0, amax.get(n))
          for n in "qkv"}
    ref, ref_lse = orc.attention(oq["q"], oq["k"], oq["v"], causal, 0.0, rows)
    # GPU path
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    if mode in ("int8_per_head", "fp8_per_head"):
        am = [torch.from_numpy(amax[n]).cuda() for n in "qkv"]
        Q, K, V = faq.quantize(dq, dk, dv, mode, layout, amax=am)
    else:
        Q, K, V = faq.quantize(dq, dk, dv, mode, layout, q_block=q_blk, kv_block=kv_blk)
    out, glse = faq.attention(Q, K, V, causal=causal, return_lse=True)
    faq.check_device_status()
    o = to_bnsd(np_of(out.float()), layout)
    sel = slice(None) if rows is None else rows
    got = o[:, :, sel, :]
    M = head_vmax(orc, oq["v"], Hq)
    mx, mean = assert_attention_close(got, ref, M, f"{mode} {layout} D={D} causal={causal}")
    gl = np_of(glse)[:, :, sel]
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.abs(gl[fin] - ref_lse[fin]).max() < 2e-3 * max(1.0, np.abs(ref_lse[fin]).max())
    return mx, mean


CASES = [
    # mode, layout, D, B, Hq, Hkv, Sq, Sk, causal
    ("fp8_per_token", "BNSD", 128, 2, 4, 2, 300, 300, True),
    ("fp8_per_token", "BNSD", 128, 1, 2, 2, 300, 300, False),
    ("fp8_per_token", "BSND", 64, 1, 4, 1, 257, 257, True),
    ("fp8_per_token", "BNSD", 128, 1, 2, 1, 100, 300, True),   # Sq < Sk, bottom-right causal
    ("fp8_block", "BSND", 128, 1, 3, 3, 300, 300, False),
    ("fp8_block", "BNSD", 64, 1, 2, 2, 200, 200, True),
    ("int8_per_head", "BNSD", 64, 1, 2, 2, 256, 256, False),
    ("int8_per_head", "BSND", 128, 2, 4, 2, 300, 300, True),
    ("mxfp4", "BNSD", 128, 1, 2, 2, 300, 300, False),
    ("mxfp4", "BSND", 128, 2, 4, 2, 257, 257, True),
    ("mxfp4", "BNSD", 128, 1, 2, 1, 100, 300, True),
    # FA PerHead FP8 and FA PerToken INT8 ("FA 量化", 该类下的模式清单)
    ("fp8_per_head", "BNSD", 128, 2, 4, 2, 300, 300, True),
    ("fp8_per_head", "BSND", 64, 1, 3, 3, 257, 257, False),
    ("int8_per_token", "BNSD", 128, 2, 4, 2, 300, 300, True),
    ("int8_per_token", "BSND", 64, 1, 2, 1, 100, 300, True),
    ("int8_per_token", "BNSD", 128, 1, 3, 3, 384, 384, False),
    # FA PerBlock MXFP8
    ("mxfp8", "BNSD", 128, 1, 2, 2, 300, 300, False),
    ("mxfp8", "BSND", 128, 2, 4, 2, 257, 257, True),
    ("mxfp8", "BNSD", 128, 1, 2, 1, 100, 300, True),
    # MX key tiles hold 112 keys: Sk an exact multiple of 112, Sk below one tile, and a causal
    # run over more tiles than the K, V' and scale rings have stages (each ring wraps)
    ("mxfp4", "BNSD", 128, 1, 2, 2, 224, 224, False),
    ("mxfp8", "BSND", 128, 1, 2, 1, 50, 50, True),
    ("mxfp4", "BNSD", 128, 1, 4, 2, 700, 700, True),
    # one query row (the second query tile of the pair is empty), one key, and an odd GQA group
    # (query row blocks paired instead of heads)
    ("mxfp4", "BNSD", 128, 2, 2, 2, 1, 300, False),
    ("mxfp8", "BNSD", 128, 1, 2, 2, 130, 1, False),
    ("mxfp4", "BSND", 128, 1, 3, 1, 260, 260, True),
]


@pytest.mark.parametrize("mode,layout,D,B,Hq,Hkv,Sq,Sk,causal", CASES)
def test_attention_matches_oracle(faq, orc, mode, layout, D, B, Hq, Hkv, Sq, Sk, causal):
    run_case(faq, orc, mode, layout, D, B, Hq, Hkv, Sq, Sk, causal, seed=len(mode) + D + Sq)


def test_fp8_block_with_non_tile_blocks(faq, orc):
    # 100-token K/V blocks: the scale varies inside a 128-key tile
    run_case(faq, orc, "fp8_block", "BNSD", 128, 1, 2, 2, 300, 300, True, seed=7, q_blk=64, kv_blk=100)


def test_rows_without_visible_keys(faq, orc):
    """Causal with Sq > Sk: the first Sq - Sk rows see no key (output 0, lse -inf)."""
    run_case(faq, orc, "fp8_per_token", "BNSD", 128, 1, 2, 2, 300, 200, True, seed=8)


def test_layouts_agree(faq, orc):
    q = wl.normal((1, 4, 200, 128), 30)
    k = wl.normal((1, 2, 200, 128), 31)
    v = wl.normal((1, 2, 200, 128), 32)
    outs = []
    for layout in ("BNSD", "BSND"):
        xs = [t if layout == "BNSD" else t.transpose(1, 2).contiguous() for t in (q, k, v)]
        Q, K, V = faq.quantize(*[x.cuda() for x in xs], "fp8_per_token", layout)
        o = faq.attention(Q, K, V, causal=True)
        outs.append(to_bnsd(np_of(o.float()), layout))
    assert np.array_equal(outs[0], outs[1])


def test_gqa_equals_repeated_kv(faq, orc):
    q = wl.normal((1, 4, 200, 128), 40).cuda()
    k = wl.normal((1, 2, 200, 128), 41).cuda()
    v = wl.normal((1, 2, 200, 128), 42).cuda()
    Q, K, V = faq.quantize(q, k, v, "fp8_per_token")
    o1 = faq.attention(Q, K, V, causal=True)
    Q2, K2, V2 = faq.quantize(q, k.repeat_interleave(2, 1).contiguous(), v.repeat_interleave(2, 1).contiguous(),
                              "fp8_per_token")
    o2 = faq.attention(Q2, K2, V2, causal=True)
    # Same arithmetic up to the fp16 rounding of P' (the two launches pair
    # query tiles differently, so the V-scale reference of a CTA can differ).
    M = float(np_of(V.scales).max() * 448.0)
    d = (o1.float() - o2.float()).abs()
    assert d.max().item() <= 5e-3 * M and d.mean().item() <= 2e-4 * M


def test_constant_v(faq, orc):
    q = wl.normal((1, 2, 300, 128), 50).cuda()
    k = wl.normal((1, 2, 300, 128), 51).cuda()
    v = torch.full((1, 2, 300, 128), 0.71875, dtype=torch.bfloat16, device="cuda")
    Q, K, V = faq.quantize(q, k, v, "fp8_per_token")
    o = faq.attention(Q, K, V, causal=True).float()
    vq = float(np_of(V.scales)[0, 0, 0]) * 448.0  # the dequantized constant
    assert torch.allclose(o, torch.full_like(o, vq), rtol=0, atol=4e-3 * vq)


def sampled_rows(Sq, seed=0, n=256):
    """Rows 0, 1, 2, the tile boundaries 127/128/255/256, the last row, and seeded random rows up
    to n in all (rows are independent, so a sample is exact where taken)."""
    fixed = [r for r in (0, 1, 2, 127, 128, 255, 256, Sq - 1) if r < Sq]
    rng = np.random.default_rng(seed)
    rest = [int(r) for r in rng.permutation(Sq) if int(r) not in fixed]
    return sorted(fixed + rest[:max(0, n - len(fixed))])


# every workload the benchmark reports a prefill number for, in its launch configuration
@pytest.mark.parametrize("name", ["fp8_prefill", "int8_tiny", "mxfp4", "int8_prefill", "fp8_head_prefill",
                                  "int8_token_prefill", "mxfp8"])
def test_full_size_workload(faq, orc, name):
    """Full-size workload in the benchmark's launch configuration, checked on 256 sampled query
    rows per head, element by element against the oracle."""
    w = wl.WORKLOADS[name]
    inp = wl.make_inputs(w)
    bits = {n: wl.bf16_bits(inp[n]) for n in "qkv"}
    amax = {}
    if w.mode in ("int8_per_head", "fp8_per_head"):
        for n in "qkv":
            amax[n] = orc.calibrate_per_head(wl.bf16_bits(inp[n + "_cal"]), w.layout)
    oq = {n: oracle_quantize(orc, w.mode, bits[n], w.layout, 0, amax.get(n)) for n in "qkv"}
    rows = sampled_rows(w.Sq)
    ref, ref_lse = orc.attention(oq["q"], oq["k"], oq["v"], w.causal, 0.0, rows)
    dev = {n: inp[n].cuda() for n in "qkv"}
    if amax:
        am = [torch.from_numpy(amax[n]).cuda() for n in "qkv"]
        Q, K, V = faq.quantize(dev["q"], dev["k"], dev["v"], w.mode, w.layout, amax=am)
    else:
        Q, K, V = faq.quantize(dev["q"], dev["k"], dev["v"], w.mode, w.layout)
    for n, G in zip("qkv", (Q, K, V)):  # the GPU's codes are the oracle's (so both see the same operands)
        assert np.array_equal(np_of(G.codes).view(np.uint8), np.ascontiguousarray(oq[n].codes).view(np.uint8)), n
    out, glse = faq.attention(Q, K, V, causal=w.causal, return_lse=True)
    faq.check_device_status()
    got = to_bnsd(np_of(out.float()), w.layout)[:, :, rows, :]
    assert_attention_close(got, ref, head_vmax(orc, oq["v"], w.Hq), name)
    gl = np_of(glse)[:, :, rows]
    assert np.abs(gl - ref_lse).max() < 2e-3 * max(1.0, np.abs(ref_lse).max())
