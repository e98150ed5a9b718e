"""Seeded synthetic inputs for the five FA-quantization workloads.

This module only draws random numbers and arranges them into the shapes,
layouts and value distributions of the workloads; it holds none of the
method's arithmetic (no scale, no rounding to a low-bit format, no
attention).  Both the oracle-side tests and the CUDA path take their inputs
from here, so the same seed gives the same bf16 bytes to both.

Workloads (shapes and distributions from the pages' three Q/K/V modes, the
rotate -> block-quant flow, and long-context decode):

  int8_tiny      B=1 H=2 S=256 D=64, BNSD, non-causal, N(0,1); per-head
                 calibration batch of the same shape from seed + 1000.
  fp8_prefill    B=2 Hq=32 Hkv=8 S=4096 D=128, BNSD, causal; Q, V ~ N(0,1);
                 K ~ N(0,1) with 4 seeded head_dim channels per kv head x20.
  rot_fp8_block  B=1 H=40 S=32768 D=128, BSND, non-causal, N(0,1); one shared
                 128x128 rotation R = bf16(Hadamard * diag(signs) / sqrt(128)).
  mxfp4          B=1 H=24 S=4096 D=128, BNSD, non-causal, Student-t df=4.
  int8_decode    B=16 Hq=32 Hkv=8 Sq=1 Sk=32768 D=128, BNSD; cached K/V and
                 Q from N(0,1); calibration batches of the same shapes from
                 seed + 1000.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Dict, Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    mode: str          # int8_per_head | fp8_per_token | fp8_block | mxfp4 | fp8_per_head | int8_per_token | mxfp8
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Sk: int
    D: int
    layout: str        # BNSD | BSND
    causal: bool
    dist: str          # normal | normal_k_outliers | student_t4
    seed: int
    rotate: bool = False
    q_block: int = 128
    kv_block: int = 256
    branch_modes: Optional[tuple] = None  # per-branch (q, k, v) modes; "float" = left unquantized

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    "int8_tiny": Workload("int8_tiny", "int8_per_head", 1, 2, 2, 256, 256, 64, "BNSD", False, "normal", 0),
    "fp8_prefill": Workload("fp8_prefill", "fp8_per_token", 2, 32, 8, 4096, 4096, 128, "BNSD", True,
                            "normal_k_outliers", 1),
    "rot_fp8_block": Workload("rot_fp8_block", "fp8_block", 1, 40, 40, 32768, 32768, 128, "BSND", False,
                              "normal", 2, rotate=True),
    "mxfp4": Workload("mxfp4", "mxfp4", 1, 24, 24, 4096, 4096, 128, "BNSD", False, "student_t4", 3),
    "int8_decode": Workload("int8_decode", "int8_per_head", 16, 32, 8, 1, 32768, 128, "BNSD", False, "normal", 4),
    # the FP8 prefill shape in the other static / dynamic modes (supplemental measurements)
    "int8_prefill": Workload("int8_prefill", "int8_per_head", 2, 32, 8, 4096, 4096, 128, "BNSD", True,
                             "normal_k_outliers", 5),
    "fp8_head_prefill": Workload("fp8_head_prefill", "fp8_per_head", 2, 32, 8, 4096, 4096, 128, "BNSD", True,
                                 "normal_k_outliers", 6),
    "int8_token_prefill": Workload("int8_token_prefill", "int8_per_token", 2, 32, 8, 4096, 4096, 128, "BNSD", True,
                                   "normal_k_outliers", 7),
    "mxfp8": Workload("mxfp8", "mxfp8", 1, 24, 24, 4096, 4096, 128, "BNSD", False, "student_t4", 8),
    # per-branch details: Q and K FP8 per token, V left unquantized (bf16), the fp8_prefill shape
    "mixed_prefill": Workload("mixed_prefill", "fp8_per_token", 2, 32, 8, 4096, 4096, 128, "BNSD", True,
                              "normal_k_outliers", 9, branch_modes=("fp8_per_token", "fp8_per_token", "float")),
}

CALIB_SEED_OFFSET = 1000
OUTLIER_CHANNELS = 4
OUTLIER_GAIN = 20.0


def shape(B: int, H: int, S: int, D: int, layout: str):
    return (B, H, S, D) if layout == "BNSD" else (B, S, H, D)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(shp, seed: int, device="cpu") -> torch.Tensor:
    """bf16 tensor of i.i.d. N(0, 1) draws."""
    g = _gen(seed, device)
    return torch.randn(shp, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def student_t4(shp, seed: int, device="cpu") -> torch.Tensor:
    """bf16 tensor of i.i.d. Student-t draws, df = 4, scale 1: z / sqrt(chi2_4 / 4)."""
    g = _gen(seed, device)
    z = torch.randn(shp, generator=g, device=device, dtype=torch.float32)
    chi2 = torch.zeros(shp, device=device, dtype=torch.float32)
    for _ in range(4):
        chi2 += torch.randn(shp, generator=g, device=device, dtype=torch.float32).square()
    return (z / torch.sqrt(chi2 / 4.0)).to(torch.bfloat16)


def outlier_channels(Hkv: int, D: int, seed: int) -> torch.Tensor:
    """[Hkv, OUTLIER_CHANNELS] seeded head_dim channel indices per kv head."""
    g = _gen(seed + 7, "cpu")
    return torch.stack([torch.randperm(D, generator=g)[:OUTLIER_CHANNELS] for _ in range(Hkv)])


def normal_k_outliers(shp, layout: str, seed: int, device="cpu") -> torch.Tensor:
    """N(0,1) keys with 4 fixed head_dim channels per kv head scaled by 20."""
    x = torch.randn(shp, generator=_gen(seed, device), device=device, dtype=torch.float32)
    H = shp[1] if layout == "BNSD" else shp[2]
    D = shp[3]
    gain = torch.ones(H, D, dtype=torch.float32)
    ch = outlier_channels(H, D, seed)
    for h in range(H):
        gain[h, ch[h]] = OUTLIER_GAIN
    gain = gain.to(device)
    if layout == "BNSD":
        x *= gain[None, :, None, :]
    else:
        x *= gain[None, None, :, :]
    return x.to(torch.bfloat16)


def rotation_signs(D: int, seed: int) -> list:
    """The seeded +-1 signs of rotation(D, seed), as a list of D ints."""
    g = _gen(seed + 11, "cpu")
    return [int(x) for x in (torch.randint(0, 2, (D,), generator=g) * 2 - 1).tolist()]


def rotation(D: int, seed: int, device="cpu") -> torch.Tensor:
    """bf16 [D, D]: Sylvester Hadamard times a seeded diagonal of +-1 signs,
    divided by sqrt(D) (orthogonal before the bf16 rounding)."""
    assert D & (D - 1) == 0
    Hm = torch.ones(1, 1, dtype=torch.float64)
    while Hm.shape[0] < D:
        Hm = torch.cat([torch.cat([Hm, Hm], 1), torch.cat([Hm, -Hm], 1)], 0)
    signs = torch.tensor(rotation_signs(D, seed), dtype=torch.float64)
    R = Hm * signs[None, :] / (D ** 0.5)
    return R.to(torch.bfloat16).to(device)


def _draw(w: Workload, which: str, shp, seed: int, device) -> torch.Tensor:
    if w.dist == "student_t4":
        return student_t4(shp, seed, device)
    if w.dist == "normal_k_outliers" and which == "k":
        return normal_k_outliers(shp, w.layout, seed, device)
    return normal(shp, seed, device)


def make_inputs(w: Workload, device="cpu", calib: bool = True) -> Dict[str, Optional[torch.Tensor]]:
    """q, k, v (bf16, the workload's layout), R for rotating workloads, and
    calibration batches (q_cal, k_cal, v_cal) for the static INT8 mode."""
    qs = shape(w.B, w.Hq, w.Sq, w.D, w.layout)
    ks = shape(w.B, w.Hkv, w.Sk, w.D, w.layout)
    out: Dict[str, Optional[torch.Tensor]] = {
        "q": _draw(w, "q", qs, 3 * w.seed + 0 + 100, device),
        "k": _draw(w, "k", ks, 3 * w.seed + 1 + 100, device),
        "v": _draw(w, "v", ks, 3 * w.seed + 2 + 100, device),
        "R": rotation(w.D, w.seed, device) if w.rotate else None,
    }
    if calib and w.mode in ("int8_per_head", "fp8_per_head"):
        c = CALIB_SEED_OFFSET
        out["q_cal"] = _draw(w, "q", qs, 3 * w.seed + 0 + 100 + c, device)
        out["k_cal"] = _draw(w, "k", ks, 3 * w.seed + 1 + 100 + c, device)
        out["v_cal"] = _draw(w, "v", ks, 3 * w.seed + 2 + 100 + c, device)
    return out


def bf16_bits(t: torch.Tensor):
    """numpy uint16 view of a bf16 tensor's bytes (CPU)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
