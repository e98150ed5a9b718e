"""Pins for the oracle's FA PerHead FP8 and FA PerToken INT8 quantizers (the wiki "FA 量化",
该类下的模式清单: per-head static INT8/FP8, per-token dynamic INT8/FP8).  Each is pinned by
the format facts (the largest element maps to the range end, half-step error bounds, exact
round trips on power-of-two scales, saturation outside the calibrated range) and by
equality with the already-pinned sibling quantizer on inputs where the two definitions
coincide."""
import numpy as np

import workloads as wl
from test_oracle_quant import bf16_from_f32, bits_of, f32, max_walk, to_bsnd


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
    # outlier channels, and a walk that puts each token's largest |x| on a channel from either end
    for x in (bits_of(wl.normal_k_outliers((2, 4, 96, 128), "BNSD", 4)), max_walk((2, 4, 96, 128), 5)):
        codes, sc = orc.quantize_int8_per_token(x)
        xf = f32(orc, x)
        assert sc.shape == (2, 4, 96)
        assert np.array_equal(sc, np.abs(xf).max(axis=-1) / np.float32(127))  # s = amax_token / 127
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
    x = wl.bf16_bits(wl.normal((2, 3, 64, 64), 35))  # B = 2, H = 3: (b, h) and (h, b) indices differ
    am = orc.calibrate_per_head(x)
    ch, sh = orc.quantize_fp8_per_head(x, am)
    ct, st = orc.quantize_int8_per_token(x)
    qh = orc.QT("fp8_per_head", ch, sh, 2, 3, 64, 64)
    qt = orc.QT("int8_per_token", ct, st, 2, 3, 64, 64)
    assert np.array_equal(orc.dequant(qh), orc.e4m3_decode(ch) * sh[None, :, None, None].astype(np.float64))
    assert np.array_equal(orc.dequant(qt), ct.astype(np.float64) * st[..., None])


# --------------------------------------------------------------- MXFP8 --
# FA PerBlock with E4M3 elements: the 组合3 rule with E4M3's largest exponent, 8
# (448 = 1.75 * 2^8), in place of E2M1's 2.

def test_mx_exponent_e4m3_brute_force(orc):
    bits = np.arange(1, 0x7F80, dtype=np.uint32)  # every positive finite bf16
    x = (bits << 16).view(np.float32)
    got = orc.mx_exponent_e4m3(x)
    # e is the integer with 2^(e+8) <= amax < 2^(e+9), clamped to [-127, 127]
    lo = np.floor(np.log2(x.astype(np.float64))).astype(np.int64) - 8
    exp = np.clip(lo, -127, 127)
    assert np.array_equal(got, exp)
    for a, e in zip(x[::997].astype(np.float64), got[::997]):  # the bracket, checked in exact arithmetic
        if -127 < e < 127:
            assert np.ldexp(1.0, int(e) + 8) <= a < np.ldexp(1.0, int(e) + 9)
    assert orc.mx_exponent_e4m3(np.array([0.0], np.float32))[0] == -127
    # the E4M3 exponent is the E2M1 exponent shifted by the two formats' emax difference
    big = (got > -127) & (got < 121)
    assert np.array_equal(got[big], orc.mx_exponent(x[big]) - 6)


def test_mxfp8_invariants(orc):
    x = bits_of(wl.student_t4((2, 3, 50, 128), 41))
    codes, e8 = orc.quantize_mxfp8(x)
    assert codes.shape == (2, 3, 50, 128) and e8.shape == (2, 3, 50, 4)
    xf = f32(orc, x).astype(np.float64)
    blocks = xf.reshape(2, 3, 50, 4, 32)
    amax = np.abs(blocks).max(-1)
    e = e8.astype(np.int64) - 127
    X = np.ldexp(1.0, np.repeat(e, 32, axis=-1))
    ratio = amax / np.ldexp(1.0, e)
    assert ((ratio >= 256) & (ratio < 512)).all()
    deq = orc.e4m3_decode(codes) * X
    # the block maximum codes to an E4M3 magnitude in [256, 448]
    top = np.take_along_axis(codes.reshape(2, 3, 50, 4, 32), np.argmax(np.abs(blocks), -1)[..., None], -1)[..., 0]
    assert np.isin(top & 0x7F, np.arange(0x78, 0x7F)).all()
    # error: half an E4M3 step (relative 2^-4 in the normal range) or saturation beyond 448
    v = np.abs(xf) / X
    bound = np.where(v <= 448, np.where(v >= 2.0 ** -6, v * 2.0 ** -4, 2.0 ** -10), v - 448) * X
    assert (np.abs(deq - xf) <= bound * (1 + 1e-9) + 1e-300).all()
    cb, eb = orc.quantize_mxfp8(to_bsnd(x), "BSND")
    assert np.array_equal(cb, to_bsnd(codes)) and np.array_equal(eb, e8)


def test_mxfp8_grid_round_trip_and_zero_block(orc):
    rng = np.random.default_rng(42)
    fin = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    big = fin[(orc.e4m3_decode(fin) >= 256)]  # magnitudes 256..448
    ok = fin[np.abs(orc.e4m3_decode(fin)) >= 2.0 ** -3]
    rows, es = [], []
    for t in range(16):
        blk = []
        for g in range(4):
            c = rng.choice(ok, 32)
            c[rng.integers(32)] = rng.choice(big)  # the block max in [256, 448]: the exponent is k exactly
            blk.append(c)
            es.append(int(rng.integers(-20, 20)))
        rows.append(np.concatenate(blk))
    codes = np.array(rows, np.uint8).reshape(1, 1, 16, 128)
    X = np.ldexp(1.0, np.repeat(np.array(es).reshape(1, 1, 16, 4), 32, axis=-1))
    x = bf16_from_f32((orc.e4m3_decode(codes) * X).astype(np.float32))
    c2, e8 = orc.quantize_mxfp8(x)
    assert np.array_equal(e8.astype(np.int64) - 127, np.array(es).reshape(1, 1, 16, 4))
    assert np.array_equal(c2, codes)
    z = np.zeros((1, 1, 2, 64), np.uint16)
    z[0, 0, 0, 3] = 0x8000
    cz, ez = orc.quantize_mxfp8(z)
    assert not ez.any() and np.array_equal(cz[0, 0, 0, 3], np.uint8(0x80)) and (cz & 0x7F == 0).all()
    q = orc.QT("mxfp8", codes, e8, 1, 1, 16, 128)
    assert np.array_equal(orc.dequant(q), orc.e4m3_decode(codes) * X)
