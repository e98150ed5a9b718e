"""The cubic 2^x of the attention kernels (ex2_poly2 in attn_common.cuh): its coefficients are
the ones the committed fit reproduces (Lawson's minimax iteration), and evaluated in fp32 the
way the kernel does it stays within 1e-4 relative error of 2^x -- below half an fp16 ulp, the
precision the probabilities are stored in."""
import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "quantized_attention_amax_b200", "csrc")


def load_fit():
    spec = importlib.util.spec_from_file_location("fit_ex2_cubic", os.path.join(CSRC, "fit_ex2_cubic.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def header_coefficients():
    src = open(os.path.join(CSRC, "attn_common.cuh")).read()
    body = src[src.index("void ex2_poly2"):]
    body = body[:body.index("\n}\n")]
    c3 = float(re.search(r"float p0 = ([0-9.e+-]+)f", body).group(1))
    rest = [float(v) for v in re.findall(r"ffma2\(p0, p1, f0, f1, ([0-9.e+-]+)f", body)]
    assert len(rest) == 3
    c2, c1, c0 = rest
    return np.array([c0, c1, c2, c3], dtype=np.float32)


def test_header_coefficients_match_the_fit():
    fit = load_fit().fit()
    hdr = header_coefficients().astype(np.float64)
    assert np.all(np.abs(hdr - fit) <= 1e-5 * np.abs(fit)), (hdr, fit)


def test_fp32_evaluation_error_bound():
    mod = load_fit()
    err = mod.max_rel_error(header_coefficients())
    assert err < 1e-4, err
    assert err < 2.0 ** -12  # half an fp16 ulp


def test_special_inputs():
    mod = load_fit()
    c = header_coefficients()
    x = np.array([0.0, 1.0, -1.0, 7.5, -125.0, -np.inf], dtype=np.float32)
    y = mod.kernel_ex2(x, c).astype(np.float64)
    ref = np.exp2(np.maximum(x.astype(np.float64), -126.0))
    assert np.all(np.abs(y[:5] / ref[:5] - 1) < 1e-4)
    assert 0.0 <= y[5] < 2.0 ** -125  # a masked score (-inf) gives a denormal-size value, read as 0
