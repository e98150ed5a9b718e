"""ctypes view of libfaq.so (include/faq.h).  Marshalling only.

The library is built in-tree by ``quantized_attention_amax_b200.build``.  If
it is missing, ``lib()`` raises: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

# FAQ_LIB=bounds selects the bounds-checked build (libfaq_bounds.so, see build.py); an absolute
# path selects another build of the same library
_sel = os.environ.get("FAQ_LIB", "")
LIB_PATH = (_sel if os.path.isabs(_sel) else
            os.path.join(os.path.dirname(os.path.abspath(__file__)),
                         "libfaq_bounds.so" if _sel == "bounds" else "libfaq.so"))

# Every entry point include/faq.h declares.
EXPORTS = (
    "fa_resolve_config",
    "fa_calibrate_per_head",
    "fa_quantize",
    "fa_rotate_quantize",
    "fa_rotate_quantize_hadamard",
    "fa_attention_quant",
    "fa_attention_workspace_size",
    "fa_attention_workspace_size_qkv",
    "fa_attention_decode_noalloc",
    "fa_decode_append",
    "fa_decode_append_workspace_size",
    "fa_check_device_status",
    "fa_status_str",
    "fa_version",
)

STATUS = {
    0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_NO_CALIBRATION",
    4: "FA_ERR_CONFIG_CONFLICT", 5: "FA_ERR_CUDA", 6: "FA_ERR_TIMEOUT", 7: "FA_ERR_WORKSPACE", 8: "FA_ERR_BOUNDS",
}


class FaTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("B", ctypes.c_int), ("H", ctypes.c_int), ("S", ctypes.c_int),
                ("D", ctypes.c_int), ("layout", ctypes.c_int)]


class FaQTensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("mode", ctypes.c_int),
                ("B", ctypes.c_int), ("H", ctypes.c_int), ("S", ctypes.c_int), ("D", ctypes.c_int),
                ("layout", ctypes.c_int), ("block_tokens", ctypes.c_int)]


class FaBranchCfg(ctypes.Structure):
    _fields_ = [("set", ctypes.c_int), ("mode", ctypes.c_int)]


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libfaq.so is not built ({LIB_PATH}); run "
                           "`python -m quantized_attention_amax_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, S, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    pT, pQ = ctypes.POINTER(FaTensor), ctypes.POINTER(FaQTensor)
    L.fa_resolve_config.argtypes = [ctypes.POINTER(FaBranchCfg), ctypes.POINTER(FaBranchCfg), ctypes.POINTER(I)]
    L.fa_calibrate_per_head.argtypes = [pT, P, P]
    L.fa_quantize.argtypes = [pT, pT, pT, I, P, P, P, pQ, pQ, pQ, P]
    L.fa_rotate_quantize.argtypes = [pT, pT, pT, P, P, I, I, pQ, pQ, pQ, P, P, P]
    L.fa_rotate_quantize_hadamard.argtypes = [pT, pT, pT, P, P, I, I, pQ, pQ, pQ, P, P, P]
    L.fa_attention_quant.argtypes = [pQ, pQ, pQ, I, F, P, P, I, P, S, P]
    L.fa_attention_decode_noalloc.argtypes = [pQ, pQ, pQ, F, P, P, I, P]
    L.fa_attention_decode_noalloc.restype = I
    L.fa_attention_workspace_size.argtypes = [pQ, pQ, I]
    L.fa_attention_workspace_size.restype = S
    L.fa_attention_workspace_size_qkv.argtypes = [pQ, pQ, pQ, I]
    L.fa_attention_workspace_size_qkv.restype = S
    L.fa_decode_append.argtypes = [pT, pT, pT, P, P, P, pQ, pQ, I, F, P, P, I, P, S, P]
    L.fa_decode_append.restype = I
    L.fa_decode_append_workspace_size.argtypes = [pT, pQ, I, I]
    L.fa_decode_append_workspace_size.restype = S
    L.fa_check_device_status.argtypes = [P]
    L.fa_status_str.argtypes = [I]
    L.fa_status_str.restype = ctypes.c_char_p
    L.fa_version.restype = ctypes.c_char_p
    for name in ("fa_resolve_config", "fa_calibrate_per_head", "fa_quantize", "fa_rotate_quantize",
                 "fa_rotate_quantize_hadamard",
                 "fa_attention_quant", "fa_check_device_status"):
        getattr(L, name).restype = I
    _lib = L
    return L
