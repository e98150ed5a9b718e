"""GPU parity for the quantize kernels: every code and every scale must equal
the oracle's, bit for bit (round-half-to-even, saturating; x / s as one IEEE
fp32 division)."""
import numpy as np
import pytest
import torch

import workloads as wl
from _gpu import bf16_from_bits, faq_module, np_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def faq():
    return faq_module()


def rand_bf16(shape, seed, dist="normal", scale=1.0):
    if dist == "t4":
        x = wl.student_t4(shape, seed).float()
    else:
        x = wl.normal(shape, seed).float()
    return (x * scale).to(torch.bfloat16)


def shp(B, H, S, D, layout):
    return (B, H, S, D) if layout == "BNSD" else (B, S, H, D)


CASES = [(layout, D, S) for layout in ("BNSD", "BSND") for D in (64, 128) for S in (1, 37, 300)]


@pytest.mark.parametrize("layout,D,S", CASES)
def test_fp8_per_token_bit_exact(faq, orc, layout, D, S):
    xs = [rand_bf16(shp(2, 3, S, D, layout), 10 + i, scale=[1.0, 30.0, 1e-3][i]) for i in range(3)]
    out = faq.quantize(*[x.cuda() for x in xs], "fp8_per_token", layout)
    torch.cuda.synchronize()
    for x, o in zip(xs, out):
        codes, scales = orc.quantize_fp8_per_token(wl.bf16_bits(x), layout)
        assert np.array_equal(np_of(o.scales), scales)
        assert np.array_equal(np_of(o.codes), codes)


@pytest.mark.parametrize("layout,D,S", CASES)
def test_mxfp4_bit_exact(faq, orc, layout, D, S):
    xs = [rand_bf16(shp(2, 3, S, D, layout), 20 + i, "t4", scale=[1.0, 1e4, 1e-5][i]) for i in range(3)]
    out = faq.quantize(*[x.cuda() for x in xs], "mxfp4", layout)
    torch.cuda.synchronize()
    for x, o in zip(xs, out):
        codes, e8 = orc.quantize_mxfp4(wl.bf16_bits(x), layout)
        assert np.array_equal(np_of(o.scales), e8)
        assert np.array_equal(np_of(o.codes), codes)


@pytest.mark.parametrize("layout,D,S", CASES)
def test_int8_calibrate_and_quantize_bit_exact(faq, orc, layout, D, S):
    cal = [rand_bf16(shp(2, 3, S, D, layout), 30 + i) for i in range(3)]
    xs = [rand_bf16(shp(2, 3, S, D, layout), 40 + i, scale=1.5) for i in range(3)]  # exceeds calibration
    amax = []
    for c in cal:
        a = faq.calibrate_per_head(c.cuda(), layout)
        a = faq.calibrate_per_head(c.cuda() * 0.5, layout, a)  # running max: a second batch changes nothing
        amax.append(a)
    out = faq.quantize(*[x.cuda() for x in xs], "int8_per_head", layout, amax=amax)
    torch.cuda.synchronize()
    for c, a, x, o in zip(cal, amax, xs, out):
        ra = orc.calibrate_per_head(wl.bf16_bits(c), layout)
        assert np.array_equal(np_of(a), ra)
        codes, scales = orc.quantize_int8_per_head(wl.bf16_bits(x), ra, layout)
        assert np.array_equal(np_of(o.scales), scales)
        assert np.array_equal(np_of(o.codes), codes)


def test_int8_per_head_every_path(faq, orc):
    """INT8 per head through each branch of the kernel: heads whose rows stay inside amax_h (no
    clamp), rows past it (saturation), non-finite data (NaN -> 0, +-inf clamped), amax_h = inf
    and NaN, scales below 2^-90 (IEEE division) and fp32-subnormal scales.  Every head is an
    exhaustive sweep of the bf16 values its range allows."""
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    fin = np.isfinite(f)
    S, D = 300, 128
    rng = np.random.default_rng(11)
    # (largest |x| of the data or None for every pattern, amax_h)
    heads = [(3.0, 3.0), (3.0, 1.0), (None, 448.0), (5.0, np.inf), (5.0, np.nan), (1e-30, 1e-30),
             (2.0 ** -130, 2.0 ** -130), (65504.0, 65504.0 * 2), (1.0, -1.0)]
    x = np.empty((1, len(heads), S, D), np.uint16)
    for h, (lim, _) in enumerate(heads):
        pool = bits if lim is None else bits[fin & (np.abs(f) <= np.float32(lim))]
        x[0, h] = np.resize(rng.permutation(pool).astype(np.uint16), S * D).reshape(S, D)
    am = np.array([a for _, a in heads], np.float32)
    o, = faq.quantize(bf16_from_bits(x), None, None, "int8_per_head", amax=[torch.from_numpy(am).cuda(), None, None])[:1]
    torch.cuda.synchronize()
    codes, scales = orc.quantize_int8_per_head(x, am)
    assert np.array_equal(np_of(o.scales), scales, equal_nan=True)
    assert np.array_equal(np_of(o.codes), codes)


@pytest.mark.parametrize("mode", ["int8_per_head", "fp8_per_head"])
def test_per_head_many_heads(faq, orc, mode):
    """More heads than the kernel's shared-memory scale table holds (the per-row path), in both
    layouts; half the heads calibrated at half their range."""
    for layout, D in (("BSND", 64), ("BNSD", 128)):
        x = rand_bf16(shp(2, 300, 7, D, layout), 77)
        a = faq.calibrate_per_head(x.cuda(), layout)
        a[::2] *= 0.5
        o, = faq.quantize(x.cuda(), None, None, mode, layout, amax=[a, None, None])[:1]
        torch.cuda.synchronize()
        fn = orc.quantize_int8_per_head if mode == "int8_per_head" else orc.quantize_fp8_per_head
        codes, scales = fn(wl.bf16_bits(x), np_of(a), layout)
        assert np.array_equal(np_of(o.scales), scales)
        assert np.array_equal(np_of(o.codes), codes)


@pytest.mark.parametrize("layout,D,S", CASES)
def test_fp8_per_head_bit_exact(faq, orc, layout, D, S):
    """FA PerHead with FP8: static scale amax_h / 448 from calibration; data past the
    calibrated range saturates to +-448."""
    cal = [rand_bf16(shp(2, 3, S, D, layout), 130 + i) for i in range(3)]
    xs = [rand_bf16(shp(2, 3, S, D, layout), 140 + i, scale=1.5) for i in range(3)]
    amax = [faq.calibrate_per_head(c.cuda(), layout) for c in cal]
    out = faq.quantize(*[x.cuda() for x in xs], "fp8_per_head", layout, amax=amax)
    torch.cuda.synchronize()
    for c, x, o in zip(cal, xs, out):
        ra = orc.calibrate_per_head(wl.bf16_bits(c), layout)
        codes, scales = orc.quantize_fp8_per_head(wl.bf16_bits(x), ra, layout)
        assert np.array_equal(np_of(o.scales), scales)
        assert np.array_equal(np_of(o.codes), codes)


@pytest.mark.parametrize("layout,D,S", CASES)
def test_int8_per_token_bit_exact(faq, orc, layout, D, S):
    """FA PerToken with INT8: dynamic scale amax_token / 127."""
    xs = [rand_bf16(shp(2, 3, S, D, layout), 150 + i, scale=[1.0, 30.0, 1e-3][i]) for i in range(3)]
    out = faq.quantize(*[x.cuda() for x in xs], "int8_per_token", layout)
    torch.cuda.synchronize()
    for x, o in zip(xs, out):
        codes, scales = orc.quantize_int8_per_token(wl.bf16_bits(x), layout)
        assert np.array_equal(np_of(o.scales), scales)
        assert np.array_equal(np_of(o.codes), codes)


@pytest.mark.parametrize("layout,D,S", CASES)
def test_mxfp8_bit_exact(faq, orc, layout, D, S):
    """FA PerBlock with MXFP8: E4M3 elements, shared exponent floor(log2 amax) - 8 per 32."""
    xs = [rand_bf16(shp(2, 3, S, D, layout), 160 + i, "t4", scale=[1.0, 1e4, 1e-5][i]) for i in range(3)]
    out = faq.quantize(*[x.cuda() for x in xs], "mxfp8", layout)
    torch.cuda.synchronize()
    for x, o in zip(xs, out):
        codes, e8 = orc.quantize_mxfp8(wl.bf16_bits(x), layout)
        assert np.array_equal(np_of(o.scales), e8)
        assert np.array_equal(np_of(o.codes), codes)


def test_mxfp8_exhaustive(faq, orc):
    maxima = [448.0, 256.0, 511.0, 3.0e38, 1e-38, 2.0 ** -130, 0.7, 100.0]
    blocks = exhaustive_rows(32, maxima, 2)
    blocks = blocks[: (len(blocks) // 4) * 4]
    x = blocks.reshape(1, 1, -1, 128)
    o, = faq.quantize(bf16_from_bits(x), None, None, "mxfp8")[:1]
    torch.cuda.synchronize()
    codes, e8 = orc.quantize_mxfp8(x)
    assert np.array_equal(np_of(o.scales), e8)
    assert np.array_equal(np_of(o.codes), codes)


def test_new_modes_exhaustive(faq, orc):
    """Every finite bf16 value through both new modes (rows of 128)."""
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    fin = bits[np.isfinite(f)].astype(np.uint16)
    x = np.resize(fin, 4 * 128 * 130).reshape(1, 4, 130, 128)
    am = np.array([448.0, 3.3e-3, 1.0, 7.5e4], np.float32)
    o, = faq.quantize(bf16_from_bits(x), None, None, "fp8_per_head", amax=[torch.from_numpy(am).cuda(), None, None])[:1]
    torch.cuda.synchronize()
    codes, scales = orc.quantize_fp8_per_head(x, am)
    assert np.array_equal(np_of(o.scales), scales) and np.array_equal(np_of(o.codes), codes)
    o, = faq.quantize(bf16_from_bits(x), None, None, "int8_per_token")[:1]
    torch.cuda.synchronize()
    codes, scales = orc.quantize_int8_per_token(x)
    assert np.array_equal(np_of(o.scales), scales) and np.array_equal(np_of(o.codes), codes)


@pytest.mark.parametrize("layout,D,S,blk", [("BSND", 128, 300, 128), ("BSND", 128, 300, 256),
                                             ("BNSD", 64, 300, 100), ("BNSD", 128, 1, 128)])
def test_fp8_block_bit_exact(faq, orc, layout, D, S, blk):
    xs = [rand_bf16(shp(1, 3, S, D, layout), 50 + i) for i in range(3)]
    out = faq.quantize(*[x.cuda() for x in xs], "fp8_block", layout, q_block=blk, kv_block=blk)
    torch.cuda.synchronize()
    for x, o in zip(xs, out):
        codes, scales = orc.quantize_fp8_block(wl.bf16_bits(x), blk, layout)
        assert np.array_equal(np_of(o.scales), scales)
        assert np.array_equal(np_of(o.codes), codes)


def exhaustive_rows(group, maxima, seed):
    """Rows (or 32-blocks) that each hold one chosen maximum and otherwise
    sweep every finite bf16 pattern not larger than it in magnitude."""
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    fin = bits[np.isfinite(f)].astype(np.uint16)
    rng = np.random.default_rng(seed)
    rows = []
    for M in maxima:
        Mb = np.array([M], np.float32).view(np.uint32)[0] >> 16
        Mv = np.array([Mb << 16], np.uint32).view(np.float32)[0]
        pool = fin[np.abs((fin.astype(np.uint32) << 16).view(np.float32)) <= Mv]
        pool = rng.permutation(pool)
        n = -(-len(pool) // (group - 1))
        pool = np.resize(pool, n * (group - 1)).reshape(n, group - 1)
        col = np.full((n, 1), Mb, np.uint16)
        rows.append(np.concatenate([col, pool], 1))
    return np.concatenate(rows, 0)


def test_fp8_per_token_exhaustive(faq, orc):
    # power-of-two scales make the e4m3 midpoints land exactly (ties); others are generic.  The
    # kernel divides by one FMA-corrected reciprocal product when s = amax / 448 >= 2^-90 and by
    # IEEE division below: maxima on both sides of amax = 448 * 2^-90 ~ 2^-81.2 cover the switch.
    maxima = [448.0, 56.0, 3.5, 1.0, 0.0546875, 3.0e38, 1e-30, 2.0 ** -126, 7.1, 0.3,
              2.0 ** -81, 2.0 ** -82, 3.6e-25, 1.7e-20]
    rows = exhaustive_rows(128, maxima, 1)
    x = rows.reshape(1, 1, -1, 128)
    o, = faq.quantize(bf16_from_bits(x), None, None, "fp8_per_token")[:1]
    torch.cuda.synchronize()
    codes, scales = orc.quantize_fp8_per_token(x)
    assert np.array_equal(np_of(o.scales), scales)
    assert np.array_equal(np_of(o.codes), codes)


def test_mxfp4_exhaustive(faq, orc):
    maxima = [6.0, 4.0, 1.5, 3.0e38, 1e-38, 2.0 ** -130, 0.7, 100.0]
    blocks = exhaustive_rows(32, maxima, 2)
    blocks = blocks[: (len(blocks) // 4) * 4]
    x = blocks.reshape(1, 1, -1, 128)
    o, = faq.quantize(bf16_from_bits(x), None, None, "mxfp4")[:1]
    torch.cuda.synchronize()
    codes, e8 = orc.quantize_mxfp4(x)
    assert np.array_equal(np_of(o.scales), e8)
    assert np.array_equal(np_of(o.codes), codes)


def test_int8_exhaustive(faq, orc):
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    fin = bits[np.isfinite(f)].astype(np.uint16)
    x = np.resize(fin, 4 * 128 * 130).reshape(1, 4, 130, 128)  # 4 heads
    am = np.array([1.0, 127.0, 3.3e-3, 7.5e4], np.float32)
    o, = faq.quantize(bf16_from_bits(x), None, None, "int8_per_head", amax=[torch.from_numpy(am).cuda(), None, None])[:1]
    torch.cuda.synchronize()
    codes, scales = orc.quantize_int8_per_head(x, am)
    assert np.array_equal(np_of(o.scales), scales)
    assert np.array_equal(np_of(o.codes), codes)


def test_zero_rows_and_empty(faq, orc):
    x = np.zeros((1, 2, 5, 128), np.uint16)
    x[0, 1, 2, 7] = 0x8000
    t = bf16_from_bits(x)
    o = faq.quantize(t, t, t, "fp8_per_token")
    m = faq.quantize(t, None, None, "mxfp4")[0]
    torch.cuda.synchronize()
    assert not np_of(o[0].codes).any() and not np_of(o[0].scales).any()
    codes, e8 = orc.quantize_mxfp4(x)
    assert np.array_equal(np_of(m.codes), codes) and np.array_equal(np_of(m.scales), e8)
    e = torch.empty((0, 2, 5, 128), dtype=torch.bfloat16, device="cuda")
    faq.quantize(e, e, e, "fp8_per_token")
    torch.cuda.synchronize()


@pytest.mark.parametrize("name", ["int8_tiny", "fp8_prefill", "mxfp4", "int8_decode"])
def test_full_size_workload_codes(faq, orc, name):
    """The workloads at full size, in the launch configuration the benchmark
    times: every code and scale bit-exact."""
    w = wl.WORKLOADS[name]
    inp = wl.make_inputs(w)
    dev = {k: (v.cuda() if v is not None else None) for k, v in inp.items()}
    if w.mode == "int8_per_head":
        amax = [faq.calibrate_per_head(dev[n + "_cal"], w.layout) for n in "qkv"]
        out = faq.quantize(dev["q"], dev["k"], dev["v"], w.mode, w.layout, amax=amax)
    else:
        out = faq.quantize(dev["q"], dev["k"], dev["v"], w.mode, w.layout)
    torch.cuda.synchronize()
    for i, n in enumerate("qkv"):
        xb = wl.bf16_bits(inp[n])
        if w.mode == "int8_per_head":
            ra = orc.calibrate_per_head(wl.bf16_bits(inp[n + "_cal"]), w.layout)
            assert np.array_equal(np_of(amax[i]), ra)
            codes, scales = orc.quantize_int8_per_head(xb, ra, w.layout)
        elif w.mode == "fp8_per_token":
            codes, scales = orc.quantize_fp8_per_token(xb, w.layout)
        else:
            codes, scales = orc.quantize_mxfp4(xb, w.layout)
        assert np.array_equal(np_of(out[i].scales), scales), n
        assert np.array_equal(np_of(out[i].codes), codes), n
