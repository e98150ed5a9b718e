"""quantized_attention_amax_b200 -- FA quantization on NVIDIA B200 (sm_100a).

Quantize Q/K/V (INT8 per-head static, FP8 E4M3 per-token dynamic, MXFP4
per-32-block, rotate -> FP8 block, FP8 per-head static, INT8 per-token
dynamic, MXFP8 per-32-block) and run flash attention on the low-bit
operands (prefill, split-KV decode, decode with the cache append fused), all in hand-written CUDA behind the C ABI of
include/faq.h (libfaq.so).  This package is the thin ctypes binding.
"""
from .api import (LAYOUTS, MODES, FaqError, QTensor, attention, attention_workspace_size, calibrate_per_head,
                  check_device_status, decode_append, dims, empty_qtensor, float_branch, quantize, resolve_config,
                  rotate_quantize, rotate_quantize_hadamard, version)

__all__ = ["LAYOUTS", "MODES", "FaqError", "QTensor", "attention", "attention_workspace_size",
           "calibrate_per_head", "check_device_status", "decode_append", "dims", "empty_qtensor", "float_branch",
           "quantize",
           "resolve_config", "rotate_quantize", "rotate_quantize_hadamard", "version"]
