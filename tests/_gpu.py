"""Helpers shared by the GPU parity tests (conversion only, no method arithmetic)."""
import numpy as np
import pytest
import torch

import workloads as wl


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def faq_module():
    require_gpu()
    from quantized_attention_amax_b200 import build
    build.build()
    import quantized_attention_amax_b200 as faq
    return faq


def np_of(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return wl.bf16_bits(t)
    return t.detach().cpu().numpy()


def oracle_qt(orc, qt):
    """An oracle QT viewing a GPU QTensor's codes and scales."""
    return orc.QT(qt.mode, np.ascontiguousarray(np_of(qt.codes)), np.ascontiguousarray(np_of(qt.scales)),
                  qt.B, qt.H, qt.S, qt.D, qt.layout, qt.block_tokens)


def bf16_from_bits(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


# Attention tolerance (relative to M_h = max |V dequantized| over the kv head
# that query head h reads): max |O - O_ref| <= 2e-2 M_h, mean <= 2e-3 M_h.
ATOL_MAX = 2e-2
ATOL_MEAN = 2e-3


def oracle_quantize(orc, mode, x_bits, layout, blk=0, amax=None):
    """The oracle's own quantization of one operand -> oracle QT."""
    from oracle import dims
    B, H, S, D = dims(x_bits.shape, layout)
    if mode == "fp8_per_token":
        c, s = orc.quantize_fp8_per_token(x_bits, layout)
    elif mode == "fp8_block":
        c, s = orc.quantize_fp8_block(x_bits, blk, layout)
    elif mode == "mxfp4":
        c, s = orc.quantize_mxfp4(x_bits, layout)
    elif mode == "int8_per_head":
        c, s = orc.quantize_int8_per_head(x_bits, amax, layout)
    elif mode == "fp8_per_head":
        c, s = orc.quantize_fp8_per_head(x_bits, amax, layout)
    elif mode == "int8_per_token":
        c, s = orc.quantize_int8_per_token(x_bits, layout)
    elif mode == "mxfp8":
        c, s = orc.quantize_mxfp8(x_bits, layout)
    else:
        raise ValueError(mode)
    return orc.QT(mode, c, s, B, H, S, D, layout, blk)


def head_vmax(orc, vq, Hq):
    """M_h for every (b, query head): max |V^| over the kv head it reads."""
    Hkv = vq.H
    m = np.zeros((vq.B, Hq))
    for b in range(vq.B):
        for hk in range(Hkv):
            mv = np.abs(orc.dequant_head(vq, b, hk)).max()
            for g in range(Hq // Hkv):
                m[b, hk * (Hq // Hkv) + g] = mv
    return m


def gpu_rows(out_bnsd: np.ndarray, rows):
    return out_bnsd[:, :, rows, :]


def assert_attention_close(got, ref, M, what=""):
    """got/ref [B, Hq, R, D]; M [B, Hq]."""
    err = np.abs(got.astype(np.float64) - ref)
    mx = err.max(axis=(2, 3)) / np.maximum(M, 1e-300)
    mean = err.mean(axis=(2, 3)) / np.maximum(M, 1e-300)
    assert mx.max() <= ATOL_MAX, f"{what}: max err {mx.max():.3e} x M_h"
    assert mean.max() <= ATOL_MEAN, f"{what}: mean err {mean.max():.3e} x M_h"
    return mx.max(), mean.max()
