"""The GPU parity tests' comparison helpers, checked on the CPU.

assert_attention_close must reject an output whose worst element misses by more than
2e-2 * M_h, or whose mean error is above 2e-3 * M_h, or that holds a NaN; it must accept one
inside both bounds.  head_vmax must give every query head the max |V| of the kv head it reads
under GQA (query head h reads kv head h // (Hq / Hkv)).
"""
import numpy as np
import pytest

import workloads as wl
from _gpu import ATOL_MAX, ATOL_MEAN, assert_attention_close, head_vmax


def test_tolerances_are_the_stated_ones():
    assert ATOL_MAX == 2e-2 and ATOL_MEAN == 2e-3


def test_head_vmax_follows_the_gqa_mapping(orc):
    B, Hq, Hkv, S, D = 2, 8, 2, 16, 64
    v = np.zeros((B, Hkv, S, D), np.float32)
    peaks = {(0, 0): 1.5, (0, 1): -3.0, (1, 0): 0.75, (1, 1): 6.0}  # bf16-exact
    for (b, hk), p in peaks.items():
        v[b, hk, 3, 5] = p
    bits = (np.ascontiguousarray(v).view(np.uint32) >> 16).astype(np.uint16)
    m = head_vmax(orc, orc.qt_float(bits, "BNSD"), Hq)
    for b in range(B):
        for h in range(Hq):
            assert m[b, h] == abs(peaks[(b, h // (Hq // Hkv))])


def case(seed=0):
    rng = np.random.default_rng(seed)
    ref = rng.standard_normal((1, 2, 32, 64))
    M = np.array([[4.0, 8.0]])
    return ref, M


def test_accepts_the_reference_and_errors_inside_both_bounds():
    ref, M = case()
    assert_attention_close(ref.copy(), ref, M)
    got = ref + 1.9e-3 * M[..., None, None] * np.sign(np.random.default_rng(1).standard_normal(ref.shape))
    got[0, 1, 7, 9] = ref[0, 1, 7, 9] + 1.9e-2 * M[0, 1]
    assert_attention_close(got, ref, M)


def test_rejects_one_element_past_the_max_bound():
    ref, M = case()
    got = ref.copy()
    got[0, 0, 31, 63] += 2.1e-2 * M[0, 0]
    with pytest.raises(AssertionError, match="max err"):
        assert_attention_close(got, ref, M)


def test_the_bound_is_per_head():
    # 3e-2 * M_0 is inside head 1's bound (M_1 = 2 M_0) but not head 0's
    ref, M = case()
    got = ref.copy()
    got[0, 0, 0, 0] += 3e-2 * M[0, 0]
    with pytest.raises(AssertionError):
        assert_attention_close(got, ref, M)
    got = ref.copy()
    got[0, 1, 0, 0] += 3e-2 * M[0, 0]
    assert_attention_close(got, ref, M)


def test_rejects_a_mean_error_past_its_bound_with_every_element_inside_the_max():
    ref, M = case()
    got = ref + 2.5e-3 * M[..., None, None]
    with pytest.raises(AssertionError, match="mean err"):
        assert_attention_close(got, ref, M)


def test_rejects_nan():
    ref, M = case()
    got = ref.copy()
    got[0, 1, 3, 3] = np.nan
    with pytest.raises(AssertionError):
        assert_attention_close(got, ref, M)


def test_bf16_bits_round_trip_used_by_the_parity_tests():
    import torch
    x = wl.normal((2, 3, 5, 64), 3)
    from _gpu import bf16_from_bits
    assert torch.equal(bf16_from_bits(wl.bf16_bits(x), device="cpu"), x)
