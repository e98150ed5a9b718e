"""The identity behind the Hadamard rotation path, pinned against the oracle's own rotation:
for R = bf16(H_D diag(sigma) / sqrt(D)) every entry is +-c with c = bf16(1 / sqrt(D)), and
x R = c * sigma * FWHT(x) elementwise, FWHT(x)_j = sum_d x_d (-1)^popcount(d & j).  The
transform here is an independent numpy butterfly; the oracle computes x R as a plain fp64 sum
of products.  Both are exact in fp64 for bf16 inputs of moderate range."""
import numpy as np
import pytest
import torch

import workloads as wl


def fwht(x):
    """Natural-order Walsh-Hadamard transform along the last axis (butterflies)."""
    y = np.array(x, dtype=np.float64, copy=True)
    D = y.shape[-1]
    h = 1
    while h < D:
        y = y.reshape(y.shape[:-1] + (D // (2 * h), 2, h))
        a, b = y[..., 0, :].copy(), y[..., 1, :].copy()
        y[..., 0, :], y[..., 1, :] = a + b, a - b
        y = y.reshape(y.shape[:-3] + (D,))
        h *= 2
    return y


def c_of(D):
    return float(torch.tensor(1.0 / np.sqrt(D), dtype=torch.float32).to(torch.bfloat16).float())


def test_fwht_matches_sylvester_matrix():
    D = 16
    H = np.array([[(-1) ** bin(i & j).count("1") for j in range(D)] for i in range(D)], dtype=np.float64)
    x = np.random.default_rng(0).integers(-1000, 1000, (5, D)).astype(np.float64)  # exact sums
    assert np.array_equal(fwht(x), x @ H)


@pytest.mark.parametrize("D,seed", [(128, 5), (64, 9)])
def test_rotation_is_scaled_signed_fwht(orc, D, seed):
    R = wl.rotation(D, seed)
    signs = np.array(wl.rotation_signs(D, seed), dtype=np.float64)
    c = c_of(D)
    assert np.all(np.abs(R.float().numpy()) == c)  # every entry is +-c
    x = wl.normal((2, 3, 50, D), seed + 1)
    xb = wl.bf16_bits(x)
    exact = orc.rotate_f64(xb, wl.bf16_bits(R), "BNSD")
    ours = c * signs * fwht(orc.bf16_bits_to_f32(xb).astype(np.float64))
    assert np.array_equal(exact, ours)
