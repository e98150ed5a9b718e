"""Pins for the oracle's FA PerHead FP8 and FA PerToken INT8 quantizers (the wiki "FA 量化",
该类下的模式清单: per-head static INT8/FP8, per-token dynamic INT8/FP8).  Each is pinned by
the format facts (the largest element maps to the range end, half-step error bounds, exact
round trips on power-of-two scales, saturation outside the calibrated range) and by
equality with the already-pinned sibling quantizer on inputs where the two definitions
coincide."""
import numpy as np

import workloads as wl
from test_oracle_quant import bf16_from_f32, bits_of, f32, to_bsnd


# ------------------------------------------------------------ FP8 per head --

def test_fp8_per_head_invariants(orc):
    x = bits_of(wl.normal((2, 4, 100, 64), 31))
    am = orc.calibrate_per_head(x)
    codes, sc = orc.quantize_fp8_per_head(x, am)
    assert sc.dtype == np.float32 and sc.shape == (4,)
    xf = f32(orc, x)
    for h in range(4):  # the largest |x| of each head codes to +-448
        i = np.unravel_index(np.argmax(np.abs(xf[:, h])), xf[:, h].shape)
        assert codes[:, h][i] in (0x7E, 0xFE)
    deq = orc.e4m3_decode(codes) * sc[None, :, None, None].astype(np.float64)
    v = np.abs(xf / sc[None, :, None, None])
    bound = np.where(v >= 2.0 ** -6, v * 2.0 ** -4, 2.0 ** -10) * sc[None, :, None, None]
    assert (np.abs(deq - xf) <= bound * (1 + 1e-6)).all()
    cb, sb = orc.quantize_fp8_per_head(to_bsnd(x), am, "BSND")
    assert np.array_equal(cb, to_bsnd(codes)) and np.array_equal(sb, sc)


def test_fp8_per_head_equals_per_token_when_every_token_reaches_the_head_max(orc):
    x = f32(orc, bits_of(wl.normal((1, 3, 40, 64), 32)))
    m = np.abs(x).max(axis=(2, 3))  # per head
    x[..., 0] = m[:, :, None]       # every token of head h now has amax = that head's max
    xb = bf16_from_f32(x.astype(np.float32))
    am = orc.calibrate_per_head(xb)
    ch, sh = orc.quantize_fp8_per_head(xb, am)
    ct, st = orc.quantize_fp8_per_token(xb)
    assert np.array_equal(st, np.broadcast_to(sh[None, :, None], st.shape))
    assert np.array_equal(ch, ct)


def test_fp8_per_head_grid_round_trip_and_saturation(orc):
    # amax = 448 * 2^-5 -> s = 2^-5 exactly; every finite E4M3 value times 2^-5 comes back
    fin = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = (orc.e4m3_decode(fin) * 2.0 ** -5).astype(np.float32)
    x = bf16_from_f32(np.resize(vals, (1, 1, 127, 4)))
    amax = np.array([448 * 2.0 ** -5], np.float32)
    codes, sc = orc.quantize_fp8_per_head(x, amax)
    assert sc[0] == np.float32(2.0 ** -5)
    back = orc.e4m3_decode(codes) * 2.0 ** -5
    assert np.array_equal(back, f32(orc, x).astype(np.float64))
    # beyond the calibrated range: saturate to +-448
    y = bf16_from_f32(np.array([[[[100.0, -100.0, 14.0, -15.0]]]], np.float32))
    c2, _ = orc.quantize_fp8_per_head(y, amax)
    assert list(c2.ravel()) == [0x7E, 0xFE, 0x7E, 0xFE]
    # a head with amax 0 codes everything to 0x00
    c3, s3 = orc.quantize_fp8_per_head(np.full((1, 1, 2, 64), 0x8000, np.uint16), np.zeros(1, np.float32))
    assert s3[0] == 0 and not c3.any()


# ----------------------------------------------------------- INT8 per token --

def test_int8_per_token_invariants(orc):
    x = bits_of(wl.normal_k_outliers((2, 4, 96, 128), "BNSD", 4))
    codes, sc = orc.quantize_int8_per_token(x)
    xf = f32(orc, x)
    assert sc.shape == (2, 4, 96)
    idx = np.argmax(np.abs(xf), axis=-1)  # the largest |x| of each token codes to +-127
    top = np.take_along_axis(codes, idx[..., None], -1)[..., 0]
    assert (np.abs(top.astype(np.int32)) == 127).all()
    deq = codes.astype(np.float64) * sc[..., None]
    assert (np.abs(deq - xf) <= sc[..., None] * (0.5 + 127 * 2.0 ** -24)).all()
    assert codes.min() >= -127  # symmetric: |x| <= amax never reaches -128
    cb, sb = orc.quantize_int8_per_token(to_bsnd(x), "BSND")
    assert np.array_equal(cb, to_bsnd(codes)) and np.array_equal(sb, sc)


def test_int8_per_token_equals_per_head_when_every_token_reaches_the_head_max(orc):
    x = f32(orc, bits_of(wl.normal((1, 3, 40, 64), 33)))
    m = np.abs(x).max(axis=(2, 3))
    x[..., 5] = -m[:, :, None]
    xb = bf16_from_f32(x.astype(np.float32))
    am = orc.calibrate_per_head(xb)
    ch, sh = orc.quantize_int8_per_head(xb, am)
    ct, st = orc.quantize_int8_per_token(xb)
    assert np.array_equal(st, np.broadcast_to(sh[None, :, None], st.shape))
    assert np.array_equal(ch, ct)


def test_int8_per_token_grid_round_trip_and_zero_token(orc):
    rng = np.random.default_rng(34)
    rows, ks = [], []
    for t in range(32):
        k = int(rng.integers(-12, 12))
        c = rng.integers(-127, 128, 64)
        c[rng.integers(64)] = 127 if rng.random() < 0.5 else -127
        rows.append(c)
        ks.append(k)
    codes = np.array(rows, np.int64).reshape(1, 1, 32, 64)
    vals = codes * np.ldexp(1.0, np.array(ks))[None, None, :, None]
    x = bf16_from_f32(vals.astype(np.float32))
    c2, sc = orc.quantize_int8_per_token(x)
    assert np.array_equal(sc.ravel(), np.ldexp(1.0, np.array(ks)).astype(np.float32))
    assert np.array_equal(c2.astype(np.int64), codes)
    z = np.zeros((1, 1, 3, 64), np.uint16)
    z[0, 0, 1, 7] = 0x8000
    cz, sz = orc.quantize_int8_per_token(z)
    assert not sz.any() and not cz.any()


def test_dequantize_new_modes_by_hand(orc):
    x = wl.bf16_bits(wl.normal((1, 2, 64, 64), 35))
    am = orc.calibrate_per_head(x)
    ch, sh = orc.quantize_fp8_per_head(x, am)
    ct, st = orc.quantize_int8_per_token(x)
    qh = orc.QT("fp8_per_head", ch, sh, 1, 2, 64, 64)
    qt = orc.QT("int8_per_token", ct, st, 1, 2, 64, 64)
    assert np.array_equal(orc.dequant(qh), orc.e4m3_decode(ch) * sh[None, :, None, None].astype(np.float64))
    assert np.array_equal(orc.dequant(qt), ct.astype(np.float64) * st[..., None])
