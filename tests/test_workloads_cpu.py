"""The seeded inputs have the five workloads' shapes and value distributions.

Shapes and layouts are those of the workload table; the same seed gives the same bytes;
K of the LLM prefill workload has exactly 4 head_dim channels per kv head scaled by 20;
the image-edit workload draws Student-t with 4 degrees of freedom (heavier tails than a
normal); the rotation is orthogonal.  Statistics are checked on small draws of the same
generators, with bounds far outside their sampling noise.
"""
import numpy as np
import pytest
import torch

import workloads as wl

TABLE = {
    # name: (mode, B, Hq, Hkv, Sq, Sk, D, layout, causal, dist)
    "int8_tiny": ("int8_per_head", 1, 2, 2, 256, 256, 64, "BNSD", False, "normal"),
    "fp8_prefill": ("fp8_per_token", 2, 32, 8, 4096, 4096, 128, "BNSD", True, "normal_k_outliers"),
    "rot_fp8_block": ("fp8_block", 1, 40, 40, 32768, 32768, 128, "BSND", False, "normal"),
    "mxfp4": ("mxfp4", 1, 24, 24, 4096, 4096, 128, "BNSD", False, "student_t4"),
    "int8_decode": ("int8_per_head", 16, 32, 8, 1, 32768, 128, "BNSD", False, "normal"),
}


@pytest.mark.parametrize("name", sorted(TABLE))
def test_workload_table(name):
    w = wl.WORKLOADS[name]
    assert (w.mode, w.B, w.Hq, w.Hkv, w.Sq, w.Sk, w.D, w.layout, w.causal, w.dist) == TABLE[name]
    if name == "rot_fp8_block":
        assert w.rotate and w.q_block == 128 and w.kv_block == 256


def test_inputs_are_deterministic_and_shaped():
    w = wl.WORKLOADS["int8_tiny"]
    a, b = wl.make_inputs(w), wl.make_inputs(w)
    for key in ("q", "k", "v", "q_cal", "k_cal", "v_cal"):
        assert a[key].dtype == torch.bfloat16 and torch.equal(a[key], b[key])
    assert tuple(a["q"].shape) == (1, 2, 256, 64)
    assert not torch.equal(a["q"], a["q_cal"])  # the calibration batch is a separate draw
    small = w.scaled(B=1, Hq=4, Hkv=2, Sq=8, Sk=12, layout="BSND")
    x = wl.make_inputs(small, calib=False)
    assert tuple(x["q"].shape) == (1, 8, 4, 64) and tuple(x["k"].shape) == (1, 12, 2, 64)


def test_k_outliers_are_four_channels_per_kv_head_scaled_by_20():
    x = wl.normal_k_outliers((1, 3, 4096, 128), "BNSD", 11).float()
    sd = x.std(dim=2)[0]  # [H, D]
    for h in range(3):
        big = (sd[h] > 5).nonzero().flatten().tolist()
        assert len(big) == wl.OUTLIER_CHANNELS == 4
        assert torch.allclose(sd[h, big], torch.full((4,), 20.0), rtol=0.1)
        rest = torch.tensor([d for d in range(128) if d not in big])
        assert torch.allclose(sd[h, rest].mean(), torch.tensor(1.0), rtol=0.05)
    # the same channels in BSND
    xb = wl.normal_k_outliers((1, 4096, 3, 128), "BSND", 11).float()
    assert torch.equal((xb.std(dim=1)[0] > 5), (sd > 5))


def test_student_t4_tails():
    x = wl.student_t4((1, 1, 1 << 16, 128), 12).float().flatten().numpy().astype(np.float64)
    # Student-t(4): mean 0, variance df / (df - 2) = 2, P(|x| > 4.604) = 0.01 (two-sided)
    assert abs(x.mean()) < 0.02
    assert abs(x.var() - 2.0) < 0.15
    assert abs((np.abs(x) > 4.604).mean() - 0.01) < 0.001
    n = wl.normal((1, 1, 1 << 16, 128), 12).float().flatten().numpy()
    assert (np.abs(n) > 4.604).mean() < 1e-4  # a normal has far thinner tails


def test_rotation_is_orthogonal_in_bf16():
    R = wl.rotation(128, 2).double()
    assert torch.allclose(R @ R.T, torch.eye(128, dtype=torch.float64), atol=1e-2)
    assert set(torch.unique(R.abs()).tolist()) == {float(torch.tensor(128 ** -0.5).to(torch.bfloat16))}
