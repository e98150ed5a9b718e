"""GPU parity for split-KV INT8 decode (Sq = 1) and its log-sum-exp combine:
every output row vs the oracle's exact attention, for several split counts,
ragged key counts and GQA group sizes, and the full-size decode workload."""
import numpy as np
import pytest
import torch

import workloads as wl
from _gpu import assert_attention_close, faq_module, head_vmax, np_of, oracle_quantize

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def faq():
    return faq_module()


def setup(orc, B, Hq, Hkv, Sk, seed, layout="BNSD", D=128):
    shp = lambda H, S: (B, H, S, D) if layout == "BNSD" else (B, S, H, D)
    q = wl.normal(shp(Hq, 1), seed)
    k = wl.normal(shp(Hkv, Sk), seed + 1)
    v = wl.normal(shp(Hkv, Sk), seed + 2)
    cal = {n: wl.normal(t.shape, seed + 10 + i) for i, (n, t) in enumerate(zip("qkv", (q, k, v)))}
    amax = {n: orc.calibrate_per_head(wl.bf16_bits(cal[n]), layout) for n in "qkv"}
    oq = {n: oracle_quantize(orc, "int8_per_head", wl.bf16_bits(t), layout, 0, amax[n])
          for n, t in zip("qkv", (q, k, v))}
    return (q, k, v), amax, oq


def gpu_decode(faq, tensors, amax, layout, splits):
    q, k, v = (t.cuda() for t in tensors)
    am = [torch.from_numpy(amax[n]).cuda() for n in "qkv"]
    Q, K, V = faq.quantize(q, k, v, "int8_per_head", layout, amax=am)
    out, lse = faq.attention(Q, K, V, causal=False, return_lse=True, num_splits=splits)
    faq.check_device_status()
    return out, lse


@pytest.mark.parametrize("B,Hq,Hkv,Sk,splits", [(2, 8, 2, 5000, 0), (2, 8, 2, 5000, 1), (1, 4, 4, 300, 3),
                                                (1, 16, 1, 1000, 0), (3, 8, 1, 129, 2), (1, 2, 2, 7, 0)])
def test_decode_matches_oracle(faq, orc, B, Hq, Hkv, Sk, splits):
    tensors, amax, oq = setup(orc, B, Hq, Hkv, Sk, seed=Sk + Hq)
    ref, ref_lse = orc.attention(oq["q"], oq["k"], oq["v"], False, 0.0)
    out, lse = gpu_decode(faq, tensors, amax, "BNSD", splits)
    got = np_of(out.float())
    assert_attention_close(got, ref, head_vmax(orc, oq["v"], Hq), f"decode splits={splits}")
    assert np.abs(np_of(lse) - ref_lse).max() < 2e-3 * max(1.0, np.abs(ref_lse).max())


def test_decode_bsnd_and_split_invariance(faq, orc):
    tensors, amax, oq = setup(orc, 2, 8, 2, 3000, seed=5, layout="BSND")
    ref, _ = orc.attention(oq["q"], oq["k"], oq["v"], False, 0.0)
    M = head_vmax(orc, oq["v"], 8)
    outs = []
    for sp in (1, 2, 5, 24):
        out, _ = gpu_decode(faq, tensors, amax, "BSND", sp)
        got = np_of(out.float()).transpose(0, 2, 1, 3)
        assert_attention_close(got, ref, M, f"splits={sp}")
        outs.append(got)
    for o in outs[1:]:
        assert np.abs(o - outs[0]).max() <= 2e-2 * M.max()


def test_full_size_decode_workload(faq, orc):
    w = wl.WORKLOADS["int8_decode"]
    inp = wl.make_inputs(w)
    amax = {n: orc.calibrate_per_head(wl.bf16_bits(inp[n + "_cal"]), w.layout) for n in "qkv"}
    oq = {n: oracle_quantize(orc, w.mode, wl.bf16_bits(inp[n]), w.layout, 0, amax[n]) for n in "qkv"}
    ref, ref_lse = orc.attention(oq["q"], oq["k"], oq["v"], False, 0.0)
    out, lse = gpu_decode(faq, (inp["q"], inp["k"], inp["v"]), amax, w.layout, 0)
    assert_attention_close(np_of(out.float()), ref, head_vmax(orc, oq["v"], w.Hq), "int8_decode")
    assert np.abs(np_of(lse) - ref_lse).max() < 2e-3 * max(1.0, np.abs(ref_lse).max())
