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
