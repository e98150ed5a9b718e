"""GPU parity for attention with per-branch modes (msModelSlim "fa3_quant 配置说明" §2.3
FA3AttentionDetails: fa_q / fa_k / fa_v each with its own QConfig; the wiki's 分支组合 note: a
branch left unset is not quantized).  Each branch is quantized on the GPU in its own mode (codes
bit-exact with the oracle's, checked elsewhere), or passed as bf16; the CUDA path (Q and K
dequantized to bf16, V' from V's own mode, bf16 QK^T on the tensor cores) is compared with the
oracle's fp64 attention on the same operands within max <= 2e-2 M_h and mean <= 2e-3 M_h."""
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


def branch(faq, orc, mode, x, layout, blk, seed):
    """(GPU operand, oracle operand) of one branch in `mode` ("float" = not quantized)."""
    bits = wl.bf16_bits(x)
    if mode == "float":
        return faq.float_branch(x.cuda(), layout), orc.qt_float(bits, layout)
    amax = None
    if mode in ("int8_per_head", "fp8_per_head"):
        cal = wl.normal(x.shape, seed + 50)
        amax = orc.calibrate_per_head(wl.bf16_bits(cal), layout)
    o = oracle_quantize(orc, mode, bits, layout, blk if mode == "fp8_block" else 0, amax)
    am = [torch.from_numpy(amax).cuda(), None, None] if amax is not None else None
    g = faq.quantize(x.cuda(), None, None, mode, layout, amax=am, q_block=blk)[0]
    assert np.array_equal(np_of(g.codes).view(np.uint8), np.ascontiguousarray(o.codes).view(np.uint8)), mode
    return g, o


def run_mixed(faq, orc, modes, layout, D, B, Hq, Hkv, Sq, Sk, causal, seed, blks=(128, 256, 256)):
    q = wl.normal(shp(B, Hq, Sq, D, layout), seed)
    k = wl.normal(shp(B, Hkv, Sk, D, layout), seed + 1)
    v = wl.normal(shp(B, Hkv, Sk, D, layout), seed + 2)
    (Q, oq), (K, ok_), (V, ov) = (branch(faq, orc, m, x, layout, b, seed + 10 * i)
                                  for i, (m, x, b) in enumerate(zip(modes, (q, k, v), blks)))
    ref, ref_lse = orc.attention(oq, ok_, ov, causal, 0.0)
    out, glse = faq.attention(Q, K, V, causal=causal, return_lse=True)
    faq.check_device_status()
    got = to_bnsd(np_of(out.float()), layout)
    mx, mean = assert_attention_close(got, ref, head_vmax(orc, ov, Hq), f"{modes} {layout} D={D} causal={causal}")
    gl = np_of(glse)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.abs(gl[fin] - ref_lse[fin]).max() < 2e-3 * max(1.0, np.abs(ref_lse[fin]).max())
    return mx, mean


MIXED = [
    # (q, k, v modes), layout, D, B, Hq, Hkv, Sq, Sk, causal
    (("fp8_per_token", "int8_per_head", "float"), "BNSD", 128, 2, 4, 2, 300, 300, True),
    (("float", "float", "float"), "BSND", 64, 1, 4, 1, 257, 257, True),          # plain bf16 attention
    (("mxfp4", "fp8_block", "mxfp8"), "BNSD", 128, 1, 2, 2, 300, 300, False),
    (("int8_per_token", "int8_per_token", "fp8_per_token"), "BSND", 128, 1, 4, 2, 100, 300, True),  # only V differs
    (("float", "fp8_per_head", "int8_per_head"), "BNSD", 64, 1, 2, 2, 200, 200, False),
    (("fp8_per_token", "fp8_per_token", "float"), "BNSD", 128, 1, 2, 2, 513, 513, True),
    (("mxfp8", "float", "mxfp4"), "BSND", 128, 1, 4, 4, 129, 129, True),
]


@pytest.mark.parametrize("modes,layout,D,B,Hq,Hkv,Sq,Sk,causal", MIXED)
def test_mixed_branches(faq, orc, modes, layout, D, B, Hq, Hkv, Sq, Sk, causal):
    run_mixed(faq, orc, modes, layout, D, B, Hq, Hkv, Sq, Sk, causal, seed=700 + Sq + D)


def test_mixed_single_query_row_and_empty_keys(faq, orc):
    """Sq = 1 with mixed branches takes the prefill path (not the INT8 decode), and Sk = 0
    gives zero rows with lse = -inf."""
    run_mixed(faq, orc, ("int8_per_head", "int8_per_head", "float"), "BNSD", 128, 2, 4, 2, 1, 300, False, seed=9)
    x = torch.zeros((1, 2, 4, 128), dtype=torch.bfloat16).cuda()
    kv = torch.zeros((1, 2, 0, 128), dtype=torch.bfloat16).cuda()
    out, lse = faq.attention(faq.float_branch(x), faq.float_branch(kv), faq.float_branch(kv), return_lse=True)
    faq.check_device_status()
    assert not np_of(out.float()).any() and np.isneginf(np_of(lse)).all()


def test_uniform_and_mixed_paths_side_by_side(faq, orc):
    """The same seeded Q, K through the uniform FP8 kernel (V FP8 too) and through the mixed path
    (V left as bf16): each within the bar against its own oracle operands."""
    a = run_mixed(faq, orc, ("fp8_per_token",) * 3, "BNSD", 128, 1, 2, 2, 256, 256, True, seed=4)
    b = run_mixed(faq, orc, ("fp8_per_token", "fp8_per_token", "float"), "BNSD", 128, 1, 2, 2, 256, 256, True,
                  seed=4)
    assert a[0] < 2e-2 and b[0] < 2e-2


def test_full_size_mixed_workload(faq, orc):
    """The benchmark's mixed-branch workload at full size (Q, K FP8 per token, V left bf16,
    B=2 Hq=32 Hkv=8 S=4096, causal), checked on 256 sampled query rows per head."""
    from test_attn_gpu import sampled_rows
    w = wl.WORKLOADS["mixed_prefill"]
    inp = wl.make_inputs(w)
    mq, mk, mv = w.branch_modes
    bits = {n: wl.bf16_bits(inp[n]) for n in "qkv"}
    oq = oracle_quantize(orc, mq, bits["q"], w.layout)
    ok_ = oracle_quantize(orc, mk, bits["k"], w.layout)
    ov = orc.qt_float(bits["v"], w.layout)
    rows = sampled_rows(w.Sq)
    ref, _ = orc.attention(oq, ok_, ov, w.causal, 0.0, rows)
    Q, K = faq.quantize(inp["q"].cuda(), inp["k"].cuda(), None, mq, w.layout)[:2]
    V = faq.float_branch(inp["v"].cuda(), w.layout)
    out = faq.attention(Q, K, V, causal=w.causal)
    faq.check_device_status()
    got = to_bnsd(np_of(out.float()), w.layout)[:, :, rows, :]
    assert_attention_close(got, ref, head_vmax(orc, ov, w.Hq), "mixed_prefill")
