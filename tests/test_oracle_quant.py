"""Pins for the oracle's quantizers and rotation: invariants the pages and the
number formats fix, exact round trips, error bounds, layout equivalence, and
library cross-checks (numpy matmul) for the rotation."""
import json
import os

import numpy as np
import pytest
import torch

import workloads as wl

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "format_constants.json")))


def bits_of(t):
    return wl.bf16_bits(t)


def f32(orc, x):
    return orc.bf16_bits_to_f32(x)


def to_bsnd(x):
    return np.ascontiguousarray(x.transpose(0, 2, 1, 3))


def max_walk(shape, seed):
    """bf16 bits of N(0,1) draws clipped to |x| <= 3.9, except that token t (the next-to-last
    axis) holds +-8 on one channel, taken alternately from both ends of D (0, D-1, 1, D-2,
    ...): the first and last channels hold some token's largest |x|, and nothing ties with it."""
    x = wl.normal(shape, seed).float().clamp(-3.9, 3.9)
    D = shape[-1]
    t = torch.arange(shape[-2])
    ch = torch.where(t % 2 == 0, (t // 2) % D, D - 1 - (t // 2) % D)
    x[..., t, ch] = torch.where(t % 2 == 0, 8.0, -8.0)
    return wl.bf16_bits(x.to(torch.bfloat16))


def bf16_from_f32(a):
    """Exact bf16 bits of float32 values that are bf16-representable."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    assert (u & 0xFFFF == 0).all()
    return (u >> 16).astype(np.uint16)


# ----------------------------------------------------------- calibration --

def test_calibrate_running_max(orc):
    a = bits_of(wl.normal((2, 3, 40, 64), 1))
    b = bits_of(wl.normal((2, 3, 40, 64), 2))
    # each head's largest |x| at an edge: head 0 in the last token of b's last batch entry,
    # head 1 in the first token of b's first entry, head 2 in the first calibration batch a
    bf = f32(orc, b).copy()
    bf[1, 0, 39, 63] = -16.0
    bf[0, 1, 0, 0] = 16.0
    af = f32(orc, a).copy()
    af[0, 2, 39, 5] = 16.0
    a, b = bf16_from_f32(af), bf16_from_f32(bf)
    am = orc.calibrate_per_head(b, "BNSD", orc.calibrate_per_head(a, "BNSD"))
    both = np.abs(np.concatenate([f32(orc, a), f32(orc, b)], axis=2))
    assert np.array_equal(am, both.max(axis=(0, 2, 3)))
    assert np.array_equal(orc.calibrate_per_head(to_bsnd(a), "BSND"), orc.calibrate_per_head(a, "BNSD"))


# ------------------------------------------------------------------ INT8 --

def test_int8_per_head_invariants(orc):
    x = bits_of(wl.normal((2, 4, 100, 64), 3))
    am = orc.calibrate_per_head(x)
    codes, sc = orc.quantize_int8_per_head(x, am)
    assert sc.dtype == np.float32 and sc.shape == (4,)
    assert np.array_equal(sc, am / np.float32(127))
    xf = f32(orc, x)
    # the element of largest |x| in each head codes to +-127
    for h in range(4):
        i = np.unravel_index(np.argmax(np.abs(xf[:, h])), xf[:, h].shape)
        assert abs(int(codes[:, h][i])) == 127
    # error bound: half a step
    deq = codes.astype(np.float64) * sc[None, :, None, None]
    # half a step, plus the fp32 rounding of x / s (at most 127 * 2^-24 steps)
    assert (np.abs(deq - xf) <= sc[None, :, None, None] * (0.5 + 127 * 2.0 ** -24)).all()
    assert codes.min() >= GOLDEN["int8_range"]["value"][0]
    # layouts agree
    cb, sb = orc.quantize_int8_per_head(to_bsnd(x), am, "BSND")
    assert np.array_equal(cb, to_bsnd(codes)) and np.array_equal(sb, sc)


def test_int8_grid_round_trip_and_out_of_calibration(orc):
    # amax = 127 * 2^-3 -> s = 2^-3 exactly; values k * 2^-3 are on the grid
    k = np.arange(-127, 128, dtype=np.float32)
    x = bf16_from_f32(np.resize(k * np.float32(0.125), (1, 1, 255, 4)))
    codes, sc = orc.quantize_int8_per_head(x, np.array([127 * 0.125], np.float32))
    assert sc[0] == 0.125
    assert np.array_equal(codes.astype(np.float32) * np.float32(0.125), f32(orc, x))
    # data outside the calibration range clamps to [-128, 127]
    y = bf16_from_f32(np.array([[[[100.0, -100.0, -16.0, -15.9375]]]], np.float32))
    c2, _ = orc.quantize_int8_per_head(y, np.array([127 * 0.125], np.float32))
    assert c2.ravel().tolist() == [127, -128, -128, -128]
    # zero calibration amax: scale 0, all codes 0
    c3, s3 = orc.quantize_int8_per_head(y, np.zeros(1, np.float32))
    assert s3[0] == 0 and not c3.any()


# --------------------------------------------------------- FP8 per token --

@pytest.mark.parametrize("walk", [False, True])
def test_fp8_per_token_invariants(orc, walk):
    # outlier channels, or a walk that puts each token's largest |x| on a channel from either end
    x = max_walk((2, 4, 96, 128), 5) if walk else bits_of(wl.normal_k_outliers((2, 4, 96, 128), "BNSD", 4))
    codes, sc = orc.quantize_fp8_per_token(x)
    xf = f32(orc, x)
    amax = np.abs(xf).max(axis=-1)
    assert sc.shape == (2, 4, 96) and np.array_equal(sc, amax / np.float32(448))
    # the max-|x| element of each token codes to +-448 (0x7E / 0xFE)
    idx = np.argmax(np.abs(xf), axis=-1)
    top = np.take_along_axis(codes, idx[..., None], -1)[..., 0]
    assert np.isin(top, [0x7E, 0xFE]).all()
    # error bound: half an E4M3 step (relative 2^-4 in the normal range,
    # absolute 2^-10 * scale in the subnormal range)
    deq = orc.e4m3_decode(codes) * sc[..., None].astype(np.float64)
    v = np.abs(xf / sc[..., None])
    bound = np.where(v >= 2.0 ** -6, v * 2.0 ** -4, 2.0 ** -10) * sc[..., None]
    assert (np.abs(deq - xf) <= bound * (1 + 1e-6)).all()
    cb, sb = orc.quantize_fp8_per_token(to_bsnd(x), "BSND")
    assert np.array_equal(cb, to_bsnd(codes)) and np.array_equal(sb, sc)


def test_fp8_grid_round_trip(orc):
    """Tokens made of E4M3 grid values times 2^k whose largest magnitude is
    448 * 2^k: the scale is exactly 2^k and every code comes back."""
    rng = np.random.default_rng(9)
    fin = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    grid = orc.e4m3_decode(fin)
    ok = np.abs(grid) >= 2.0 ** -3  # keep x = grid * 2^k inside the bf16 normal range for k >= -120
    cand = fin[ok]
    rows = []
    ks = []
    for t in range(64):
        k = int(rng.integers(-20, 20))
        c = rng.choice(cand, 64)
        c[rng.integers(64)] = 0x7E if rng.random() < 0.5 else 0xFE
        rows.append(c)
        ks.append(k)
    codes = np.array(rows, np.uint8).reshape(1, 1, 64, 64)
    vals = orc.e4m3_decode(codes) * np.ldexp(1.0, np.array(ks))[None, None, :, None]
    x = bf16_from_f32(vals.astype(np.float32))
    c2, sc = orc.quantize_fp8_per_token(x)
    assert np.array_equal(sc.ravel(), np.ldexp(1.0, np.array(ks)).astype(np.float32))
    assert np.array_equal(c2, codes)


def test_fp8_zero_token(orc):
    x = np.zeros((1, 1, 3, 64), np.uint16)
    x[0, 0, 1, 5] = 0x8000  # -0.0
    codes, sc = orc.quantize_fp8_per_token(x)
    assert not sc.any() and not codes.any()


# ----------------------------------------------------------------- MXFP4 --

def test_mxfp4_invariants(orc):
    assert GOLDEN["mxfp4_block_elems"]["value"] == 32
    x = bits_of(wl.student_t4((2, 3, 50, 128), 5))
    codes, e8 = orc.quantize_mxfp4(x)
    assert codes.shape == (2, 3, 50, 64) and e8.shape == (2, 3, 50, 4)
    xf = f32(orc, x).astype(np.float64)
    blocks = xf.reshape(2, 3, 50, 4, 32)
    amax = np.abs(blocks).max(-1)
    e = e8.astype(np.int64) - 127
    # E8M0 exponent = floor(log2 amax) - emax, emax = 2
    assert np.array_equal(e, np.floor(np.log2(amax)).astype(np.int64) - GOLDEN["e2m1_emax"]["value"])
    lo, hi = codes & 15, codes >> 4
    nib = np.stack([lo, hi], -1).reshape(2, 3, 50, 128)
    deq = orc.e2m1_decode(nib) * np.ldexp(1.0, np.repeat(e, 32, axis=-1))
    # the block maximum codes to magnitude 4 or 6
    bmax_idx = np.argmax(np.abs(blocks), -1)
    topcode = np.take_along_axis(nib.reshape(2, 3, 50, 4, 32), bmax_idx[..., None], -1)[..., 0] & 7
    assert np.isin(topcode, [6, 7]).all()
    # error bound: half a grid step, or saturation beyond 6
    v = np.abs(xf) / np.ldexp(1.0, np.repeat(e, 32, axis=-1))
    step = np.where(v < 2, 0.5, np.where(v < 4, 1.0, 2.0))
    bound = np.where(v <= 6, step / 2, v - 6) * np.ldexp(1.0, np.repeat(e, 32, axis=-1))
    assert (np.abs(deq - xf) <= bound + 1e-300).all()
    cb, eb = orc.quantize_mxfp4(to_bsnd(x), "BSND")
    assert np.array_equal(cb, to_bsnd(codes)) and np.array_equal(eb, e8)


def test_mxfp4_grid_round_trip(orc):
    rng = np.random.default_rng(10)
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    nib = rng.integers(0, 16, (1, 1, 8, 64))
    nib[..., ::32] = rng.choice([6, 7, 14, 15], nib[..., ::32].shape)  # block max 4 or 6
    e = rng.integers(-30, 30, (1, 1, 8, 2))
    vals = np.where(nib & 8, -1, 1) * mags[nib & 7] * np.ldexp(1.0, np.repeat(e, 32, -1))
    x = bf16_from_f32(vals.astype(np.float32))
    codes, e8 = orc.quantize_mxfp4(x)
    assert np.array_equal(e8.astype(np.int64) - 127, e)
    got = np.stack([codes & 15, codes >> 4], -1).reshape(nib.shape)
    # +0 and -0 both decode to 0; compare values
    assert np.array_equal(orc.e2m1_decode(got), orc.e2m1_decode(nib.astype(np.uint8)))


def test_mxfp4_zero_block(orc):
    x = np.zeros((1, 1, 1, 64), np.uint16)
    codes, e8 = orc.quantize_mxfp4(x)
    assert e8.tolist() == [[[[0, 0]]]] and not codes.any()


# ------------------------------------------------------------- FP8 block --

def test_fp8_block_invariants(orc):
    assert GOLDEN["q_block_tokens"]["value"] == 128 and GOLDEN["kv_block_tokens"]["value"] == 256
    x = bits_of(wl.normal((2, 300, 3, 64), 6))  # BSND, ragged last block, B = 2 and H = 3
    for blk in (128, 256):
        codes, sc = orc.quantize_fp8_block(x, blk, "BSND")
        nblk = -(-300 // blk)
        assert sc.shape == (2, 3, nblk)
        xf = f32(orc, x)  # [B, S, H, D]
        for b in range(2):
            for h in range(3):
                for g in range(nblk):
                    blkx = xf[b, g * blk:(g + 1) * blk, h]
                    assert sc[b, h, g] == np.abs(blkx).max() / np.float32(448)
                    i = np.unravel_index(np.argmax(np.abs(blkx)), blkx.shape)
                    assert codes[b, g * blk:(g + 1) * blk, h][i] in (0x7E, 0xFE)
        # a block of exactly one token per block is per-token quantization
    c1, s1 = orc.quantize_fp8_block(x, 1, "BSND")
    c2, s2 = orc.quantize_fp8_per_token(x, "BSND")
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


# -------------------------------------------------------------- rotation --

def test_rotate_matches_numpy_matmul(orc):
    x = bits_of(wl.normal((1, 2, 33, 64), 7))
    R = bits_of(wl.normal((64, 64), 8))  # deliberately not symmetric
    got = orc.rotate_f64(x, R)
    ref = f32(orc, x).astype(np.float64) @ f32(orc, R).astype(np.float64)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)
    # and the bf16 output is the nearest bf16 of that sum
    assert np.array_equal(orc.rotate(x, R), orc.f64_to_bf16(got))
    # rounded once: 1 + 2^-8 + 2^-30 lies just above the midpoint of 1 and 1 + 2^-7 and rounds
    # up, where a detour through fp32 (1 + 2^-8, a tie) would round to even, 1
    xo = np.zeros((1, 1, 1, 64), np.float32)
    xo[0, 0, 0, :3] = [1.0, 2.0 ** -8, 2.0 ** -30]
    Ro = np.zeros((64, 64), np.float32)
    Ro[:3, 0] = 1.0
    assert f32(orc, orc.rotate(bf16_from_f32(xo), bf16_from_f32(Ro)))[0, 0, 0, 0] == 1.0 + 2.0 ** -7
    xb = to_bsnd(x)
    assert np.array_equal(orc.rotate(xb, R, "BSND"), to_bsnd(orc.rotate(x, R)))


def test_rotate_identity_and_signed_permutation(orc):
    x = bits_of(wl.normal((1, 300, 2, 64), 9))  # BSND
    eye = bf16_from_f32(np.eye(64, dtype=np.float32))
    assert np.array_equal(orc.rotate(x, eye, "BSND"), x)
    rng = np.random.default_rng(11)
    perm = rng.permutation(64)
    sign = rng.choice([-1.0, 1.0], 64)
    P = np.zeros((64, 64), np.float32)
    P[perm, np.arange(64)] = sign  # (x P)[:, j] = sign[j] * x[:, perm[j]]
    xr = orc.rotate(x, bf16_from_f32(P), "BSND")
    expect = x[..., perm] ^ np.where(sign < 0, 0x8000, 0).astype(np.uint16)
    assert np.array_equal(xr, expect)
    for blk in (128, 256):
        c0, s0 = orc.quantize_fp8_block(x, blk, "BSND")
        c1, s1 = orc.quantize_fp8_block(xr, blk, "BSND")
        assert np.array_equal(s0, s1)
        assert np.array_equal(c1, c0[..., perm] ^ np.where(sign < 0, 0x80, 0).astype(np.uint8))


def test_rotation_preserves_qk(orc):
    """With an exactly orthogonal R (normalised Hadamard for D = 64: entries
    +-1/8, exact in bf16), (QR)(KR)^T = QK^T."""
    D = 64
    R = wl.rotation(D, seed=3)
    Rf = R.float().numpy().astype(np.float64)
    assert np.array_equal(Rf @ Rf.T, np.eye(D))
    q = bits_of(wl.normal((1, 1, 20, D), 12))
    k = bits_of(wl.normal((1, 1, 30, D), 13))
    Rb = wl.bf16_bits(R)
    qr, kr = orc.rotate_f64(q, Rb), orc.rotate_f64(k, Rb)
    s0 = f32(orc, q)[0, 0].astype(np.float64) @ f32(orc, k)[0, 0].astype(np.float64).T
    s1 = qr[0, 0] @ kr[0, 0].T
    assert np.allclose(s0, s1, rtol=0, atol=1e-12 * np.abs(s0).max())


def test_workload_rotation_is_signed_scaled_hadamard():
    R = wl.rotation(128, seed=2).float().numpy()
    assert np.all(np.abs(R) == np.float32(0.08837890625))
    Rs = np.sign(R)
    assert np.array_equal(Rs @ Rs.T, 128 * np.eye(128))
