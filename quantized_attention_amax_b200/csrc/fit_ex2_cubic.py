"""Fit of the cubic that the attention kernels use for 2^x on the FMA pipe (ex2_poly2 in
attn_common.cuh), and its error check in fp32.  numpy only.

    python fit_ex2_cubic.py          # prints the coefficients and the error bounds

The kernel writes x = n + f with n = rint(x) and f in [-0.5, 0.5], evaluates a cubic p(f) by
Horner's rule in fp32 and adds n to the exponent field of p(f).  The cubic is chosen to minimise
the largest relative error |p(f) / 2^f - 1| over [-0.5, 0.5]: Lawson's algorithm (C. L. Lawson,
"Contributions to the theory of linear least maximum approximation", UCLA thesis, 1961) finds that
minimax solution as the limit of weighted least-squares fits whose weights are multiplied, each
step, by the current pointwise error.
"""
import numpy as np

GRID = 20001       # sample points on [-0.5, 0.5]
STEPS = 300        # Lawson iterations


def fit(grid: int = GRID, steps: int = STEPS) -> np.ndarray:
    """Coefficients c0..c3 (fp64) of the cubic of least maximum relative error for 2^f."""
    f = np.linspace(-0.5, 0.5, grid)
    target = np.exp2(f)
    # relative error r = (sum_k c_k f^k) / 2^f - 1: linear in c, rows scaled by 1 / 2^f
    basis = np.vander(f, 4, increasing=True) / target[:, None]
    weight = np.full(grid, 1.0 / grid)
    coef = None
    for _ in range(steps):
        sw = np.sqrt(weight)
        coef, *_ = np.linalg.lstsq(basis * sw[:, None], sw, rcond=None)
        err = np.abs(basis @ coef - 1.0)
        weight = weight * err
        weight /= weight.sum()
    return coef


def kernel_ex2(x: np.ndarray, coef32: np.ndarray) -> np.ndarray:
    """The kernel's steps in fp32: clamp at -126, n = rint(x) through the 1.5 * 2^23 trick,
    f = x - n, Horner with fused multiply-adds (emulated by one rounding of the fp64 product-sum),
    then n added to the exponent field."""
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    j = (x + magic).astype(np.float32)
    n = (j - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = np.full_like(f, coef32[3])
    for c in (coef32[2], coef32[1], coef32[0]):
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(c)).astype(np.float32)
    bits = p.view(np.int32) + (j.view(np.int32) << 23)
    return bits.view(np.float32)


def max_rel_error(coef32: np.ndarray, lo: float = -100.0, hi: float = 8.0, n: int = 2_000_001) -> float:
    """Largest relative error of the fp32 evaluation against 2^x over [lo, hi] (normal results)."""
    x = np.linspace(lo, hi, n).astype(np.float32)
    got = kernel_ex2(x, coef32).astype(np.float64)
    return float(np.max(np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)))


if __name__ == "__main__":
    c = fit()
    c32 = c.astype(np.float32)
    f = np.linspace(-0.5, 0.5, GRID)
    print("coefficients c0..c3:", ", ".join(f"{float(v):.9e}" for v in c32))
    print("minimax relative error (fp64 cubic):", float(np.abs(np.polyval(c[::-1], f) / np.exp2(f) - 1).max()))
    print("max relative error of the fp32 evaluation on [-100, 8]:", max_rel_error(c32))
    print("half an fp16 ulp:", 2.0 ** -12)
