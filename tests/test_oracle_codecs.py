"""Pins for the oracle's scalar codecs.

Each codec is checked against something other than itself: a brute-force
nearest-representable-value search over every code (values decoded here from
the format's bit-field definition), the independent ml_dtypes library, and
the format constants the pages print (tests/golden/format_constants.json).
"""
import json
import math
import os

import ml_dtypes
import numpy as np
import pytest

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "format_constants.json")))


def all_finite_bf16_f32():
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    return f[np.isfinite(f)]


def e4m3_table():
    """Value of every float8_e4m3fn code from the bit fields (bias 7, 3 mantissa
    bits, subnormals at exponent field 0, S.1111.111 = NaN)."""
    vals = np.empty(256)
    for c in range(256):
        s, e, m = c >> 7, (c >> 3) & 15, c & 7
        if e == 15 and m == 7:
            v = math.nan
        elif e == 0:
            v = m / 8 * 2.0 ** -6
        else:
            v = (1 + m / 8) * 2.0 ** (e - 7)
        vals[c] = -v if s else v
    return vals


def brute_nearest(v, codes, values):
    """Nearest value among (codes, values) to each v; ties go to the even code.
    Returns chosen codes.  `values` are non-negative magnitudes."""
    a = np.abs(v.astype(np.float64))[:, None]
    dist = np.abs(a - values[None, :])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    # among tied candidates prefer the one with an even code (mantissa lsb 0)
    even = (codes[None, :] & 1) == 0
    pick_even = cand & even
    has_even = pick_even.any(axis=1)
    idx = np.where(has_even, np.argmax(pick_even, axis=1), np.argmax(cand, axis=1))
    return codes[idx]


# ------------------------------------------------------------------ E4M3 --

def test_e4m3_max_is_the_pages_448(orc):
    assert GOLDEN["e4m3_max"]["value"] == 448
    tab = e4m3_table()
    assert np.nanmax(tab) == 448.0
    assert orc.e4m3_decode(orc.e4m3_encode(np.array([1e30, 449.0, 10000.0], np.float32))).tolist() == [448.0] * 3
    assert orc.e4m3_encode(np.array([-1e30], np.float32))[0] == 0xFE


def test_e4m3_decode_matches_bitfields_and_ml_dtypes(orc):
    tab = e4m3_table()
    ours = orc.e4m3_decode(np.arange(256, dtype=np.uint8))
    fin = ~np.isnan(tab)
    assert np.array_equal(ours[fin], tab[fin])
    assert np.isnan(ours[~fin]).all()
    lib = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    assert np.array_equal(ours[fin], lib[fin])


def test_e4m3_encode_brute_force(orc):
    tab = e4m3_table()
    pos = np.arange(0, 127, dtype=np.int64)           # 0x00..0x7E, finite magnitudes
    vals = tab[pos]
    rng = np.random.default_rng(5)
    v = np.concatenate([
        all_finite_bf16_f32(),
        rng.standard_normal(200000).astype(np.float32) * np.float32(50),
        (vals[:-1] + vals[1:]).astype(np.float32) / 2,     # exact midpoints (ties)
        np.array([448, 460, 463.99, 464, 465, 479, 480, 1e5, 2.0 ** -10, 2.0 ** -9 * 0.5], np.float32),
    ]).astype(np.float32)
    v = np.concatenate([v, -v])
    got = orc.e4m3_encode(v)
    # saturating reading: every finite magnitude above 448 encodes as 448
    a = np.abs(v.astype(np.float64))
    expect_mag = np.where(a > 448, 0x7E, 0)
    inr = a <= 448
    for chunk in np.array_split(np.nonzero(inr)[0], 64):
        expect_mag[chunk] = brute_nearest(v[chunk], pos, vals)
    expect = expect_mag | np.where(np.signbit(v), 0x80, 0)
    assert np.array_equal(got, expect.astype(np.uint8))


def test_e4m3_encode_matches_ml_dtypes_in_range(orc):
    v = all_finite_bf16_f32()
    v = v[np.abs(v) < 464]  # ml_dtypes turns >= the overflow midpoint into NaN; ours saturates
    got = orc.e4m3_encode(v)
    lib = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(got, lib)


def test_e4m3_all_finite_codes_round_trip(orc):
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = orc.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(orc.e4m3_encode(vals), codes)


# ------------------------------------------------------------------ E2M1 --

E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def test_e2m1_constants_are_the_pages(orc):
    assert GOLDEN["e2m1_max"]["value"] == 6 and GOLDEN["e2m1_emax"]["value"] == 2
    # largest magnitude 6 = 1.5 * 2^emax
    assert orc.e2m1_decode(np.arange(16, dtype=np.uint8)).max() == 6.0 == 1.5 * 2 ** 2
    assert orc.e2m1_encode(np.array([7.0, 100.0, -1e9], np.float32)).tolist() == [7, 7, 15]


def test_e2m1_decode_matches_ml_dtypes(orc):
    ours = orc.e2m1_decode(np.arange(16, dtype=np.uint8))
    # ml_dtypes stores one e2m1 per byte, value in the low nibble
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(ours, lib)


def test_e2m1_encode_brute_force(orc):
    codes = np.arange(8)
    rng = np.random.default_rng(6)
    v = np.concatenate([
        all_finite_bf16_f32(),
        rng.standard_normal(100000).astype(np.float32) * 3,
        np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0, 8.0], np.float32),
    ])
    v = np.concatenate([v, -v])
    got = orc.e2m1_encode(v)
    a = np.abs(v.astype(np.float64))
    mag = np.where(a > 6, 7, 0)
    inr = np.nonzero(a <= 6)[0]
    for chunk in np.array_split(inr, 32):
        mag[chunk] = brute_nearest(v[chunk], codes, E2M1_MAG)
    expect = (mag | np.where(np.signbit(v), 8, 0)).astype(np.uint8)
    assert np.array_equal(got, expect)
    # worked ties from round-half-to-even on the grid
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    assert orc.e2m1_decode(orc.e2m1_encode(ties)).tolist() == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]


def test_e2m1_matches_ml_dtypes(orc):
    v = all_finite_bf16_f32()
    got = orc.e2m1_encode(v)
    lib = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 15
    assert np.array_equal(got, lib)


# ------------------------------------------------------------------ INT8 --

def test_int8_range_is_the_pages(orc):
    lo, hi = GOLDEN["int8_range"]["value"]
    got = orc.int8_encode(np.array([1e6, -1e6, 127.5, -128.5, -127.5, 126.5], np.float32))
    assert got.tolist() == [hi, lo, hi, lo, -128, 126]


def test_int8_exhaustive_bf16_times_scales(orc):
    """x / s in IEEE fp32 (numpy), then nearest integer by comparing the two
    neighbouring integers (ties to the even one), clamped to [-128, 127]."""
    x = all_finite_bf16_f32()
    rng = np.random.default_rng(7)
    amaxes = np.concatenate([[127.0, 1.0, 3.3], rng.uniform(0.5, 8, 5)]).astype(np.float32)
    for amax in amaxes:
        s = np.float32(amax) / np.float32(127.0)
        with np.errstate(over="ignore"):
            v = (x / s).astype(np.float32)
        v = v[np.isfinite(v)]
        got = orc.int8_encode(v).astype(np.int64)
        vd = v.astype(np.float64)
        lo = np.floor(vd)
        hi = lo + 1
        dlo, dhi = vd - lo, hi - vd
        pick = np.where(dlo < dhi, lo, np.where(dhi < dlo, hi, np.where(lo % 2 == 0, lo, hi)))
        expect = np.clip(pick, -128, 127).astype(np.int64)
        assert np.array_equal(got, expect), amax


# ------------------------------------------------------------------ E8M0 --

def test_mx_exponent_brute_force(orc):
    """e is the integer with 2^(e+2) <= amax < 2^(e+3), clamped to [-127, 127]."""
    x = all_finite_bf16_f32()
    x = x[x > 0]
    got = orc.mx_exponent(x)
    expect = []
    for a in x.astype(np.float64):
        e = -200
        while math.ldexp(1.0, e + 3) <= a:
            e += 1
        # walk from below: the first e with 2^(e+3) > a, then check the lower bound
        assert math.ldexp(1.0, e + 2) <= a or e == -200
        expect.append(min(max(e, -127), 127))
    assert np.array_equal(got, np.array(expect))
    assert orc.mx_exponent(np.array([0.0], np.float32))[0] == -127
    # emax = 2: the block maximum lands in [4, 8) times 2^e
    e = orc.mx_exponent(x)
    ratio = x.astype(np.float64) / np.ldexp(1.0, e)
    big = e > -127
    assert ((ratio[big] >= 4) & (ratio[big] < 8)).all()


def test_mx_exponent_matches_ml_dtypes_floor(orc):
    """ml_dtypes' float8_e8m0fnu conversion rounds toward the lower power of
    two for positive normal inputs below the midpoint; compare the exponent
    of 2^floor(log2 a) on exact powers of two and on values just above."""
    e = np.arange(-120, 120)
    a = np.ldexp(1.0, e).astype(np.float32)
    lib = a.astype(ml_dtypes.float8_e8m0fnu).view(np.uint8).astype(np.int64) - 127
    assert np.array_equal(orc.mx_exponent(a), lib - 2)


# ------------------------------------------------------------------ bf16 --

def test_f64_to_bf16_nearest_by_search(orc):
    bits = np.arange(0x7F80, dtype=np.uint32)              # all finite non-negative bf16
    grid = (bits << 16).view(np.float32).astype(np.float64)
    rng = np.random.default_rng(8)
    v = np.concatenate([rng.standard_normal(50000) * 10 ** rng.uniform(-30, 30, 50000),
                        (grid[:-1] + grid[1:]) / 2,         # exact ties
                        grid[::97]])
    got = orc.f64_to_bf16(v)
    a = np.abs(v)
    i = np.clip(np.searchsorted(grid, a), 1, len(grid) - 1)
    lo, hi = grid[i - 1], grid[i]
    pick = np.where(a - lo < hi - a, i - 1, np.where(hi - a < a - lo, i,
                                                     np.where((i - 1) % 2 == 0, i - 1, i)))
    pick = np.where(a == grid[i], i, pick)
    expect = bits[pick].astype(np.uint16) | np.where(np.signbit(v), 0x8000, 0).astype(np.uint16)
    assert np.array_equal(got, expect)


# ------------------------------------------------------- non-finite values --
# The method's inputs are finite, but the codecs' edges are part of their definitions:
# IEEE round-to-nearest carries bf16 past the largest finite value to infinity; E4M3
# (float8_e4m3fn) has no infinity, saturates finite values at 448 and keeps NaN as
# S.1111.111; E2M1 has neither infinity nor NaN and saturates at 6; INT8 clamps to
# [-128, 127] and takes NaN to 0.

def test_bf16_rounds_past_the_largest_finite_value_to_infinity(orc):
    top = float((np.uint32(0x7F7F) << 16).view(np.float32))  # largest finite bf16, odd mantissa
    mid = (top + 2.0 ** 128) / 2                              # the tie goes to the even side: infinity
    got = orc.f64_to_bf16(np.array([top, mid, np.nextafter(mid, 0), 1e39, -1e39, -mid, np.inf, -np.inf]))
    assert got.tolist() == [0x7F7F, 0x7F80, 0x7F7F, 0x7F80, 0xFF80, 0xFF80, 0x7F80, 0xFF80]


def test_e4m3_non_finite(orc):
    got = orc.e4m3_encode(np.array([np.inf, -np.inf, np.nan, 1e30, -1e30], np.float32))
    assert got.tolist() == [0x7E, 0xFE, 0x7F, 0x7E, 0xFE]
    assert np.isnan(orc.e4m3_decode(np.array([0x7F, 0xFF], np.uint8))).all()


def test_e2m1_non_finite(orc):
    got = orc.e2m1_encode(np.array([np.inf, -np.inf, 1e30, -1e30], np.float32))
    assert got.tolist() == [7, 15, 7, 15]


def test_int8_non_finite(orc):
    got = orc.int8_encode(np.array([np.inf, -np.inf, np.nan], np.float32))
    assert got.tolist() == [127, -128, 0]
