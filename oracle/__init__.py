"""The oracle for FA quantization: numpy-level access to liboracle.so.

TEST INFRASTRUCTURE ONLY.  Only tests/, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  It
shares no code with ``quantized_attention_amax_b200`` and imports nothing
from it.

Tensors are numpy arrays: bf16 data as ``uint16`` bit patterns shaped
``[B, H, S, D]`` (layout ``"BNSD"``) or ``[B, S, H, D]`` (layout ``"BSND"``).
Every function cites the page passage it follows in the C source
(oracle/faq_oracle.c).
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

from . import build as _build

LAYOUTS = {"BNSD": 0, "BSND": 1}
MODES = {"float": 0, "int8_per_head": 1, "fp8_per_token": 2, "mxfp4": 3, "fp8_block": 4, "fp8_per_head": 5,
         "int8_per_token": 6, "mxfp8": 7}

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        Z = ctypes.c_size_t
        L.orc_bf16_to_f32.restype = ctypes.c_float
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_f64_to_bf16.restype = ctypes.c_uint16
        L.orc_f64_to_bf16.argtypes = [ctypes.c_double]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_encode.argtypes = [ctypes.c_float]
        L.orc_e4m3_decode.restype = ctypes.c_double
        L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.orc_e2m1_encode.restype = ctypes.c_uint8
        L.orc_e2m1_encode.argtypes = [ctypes.c_float]
        L.orc_e2m1_decode.restype = ctypes.c_double
        L.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.orc_int8_encode.restype = ctypes.c_int8
        L.orc_int8_encode.argtypes = [ctypes.c_float]
        L.orc_mx_exponent.restype = ctypes.c_int
        L.orc_mx_exponent.argtypes = [ctypes.c_float]
        for name in ("orc_e4m3_encode_n", "orc_e2m1_encode_n", "orc_int8_encode_n",
                     "orc_mx_exponent_n", "orc_mx_exponent_e4m3_n", "orc_f64_to_bf16_n"):
            getattr(L, name).restype = None
            getattr(L, name).argtypes = [P, P, Z]
        L.orc_calibrate_per_head.argtypes = [P, I, I, I, I, I, P]
        L.orc_quantize_int8_per_head.argtypes = [P, I, I, I, I, I, P, P, P]
        L.orc_quantize_fp8_per_token.argtypes = [P, I, I, I, I, I, P, P]
        L.orc_quantize_fp8_per_head.argtypes = [P, I, I, I, I, I, P, P, P]
        L.orc_quantize_int8_per_token.argtypes = [P, I, I, I, I, I, P, P]
        L.orc_quantize_mxfp4.argtypes = [P, I, I, I, I, I, P, P]
        L.orc_quantize_mxfp8.argtypes = [P, I, I, I, I, I, P, P]
        L.orc_rotate_f64.argtypes = [P, I, I, I, I, I, P, P]
        L.orc_rotate.argtypes = [P, I, I, I, I, I, P, P]
        L.orc_quantize_fp8_block.argtypes = [P, I, I, I, I, I, I, P, P]
        L.orc_dequant_head.argtypes = [ctypes.POINTER(_OrcQT), I, I, P]
        L.orc_attention.argtypes = [ctypes.POINTER(_OrcQT)] * 3 + [I, ctypes.c_double, P, I, P, P]
        L.orc_num_threads.restype = I
        _lib = L
    return _lib


class _OrcQT(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("B", ctypes.c_int), ("H", ctypes.c_int), ("S", ctypes.c_int), ("D", ctypes.c_int),
                ("layout", ctypes.c_int), ("blk", ctypes.c_int)]


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def dims(shape: Sequence[int], layout: str):
    """(B, H, S, D) of a tensor of the given shape in the given layout."""
    if layout == "BNSD":
        B, H, S, D = shape
    else:
        B, S, H, D = shape
    return B, H, S, D


def num_threads() -> int:
    return lib().orc_num_threads()


# ---------------------------------------------------------------- codecs ---

def bf16_bits_to_f32(x: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(x, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e4m3_encode_n(_ptr(v), _ptr(out), v.size)
    return out


def e4m3_decode(c: np.ndarray) -> np.ndarray:
    L = lib()
    table = np.array([L.orc_e4m3_decode(i) for i in range(256)], dtype=np.float64)
    return table[np.asarray(c, dtype=np.uint8)]


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().orc_e2m1_encode_n(_ptr(v), _ptr(out), v.size)
    return out


def e2m1_decode(c: np.ndarray) -> np.ndarray:
    L = lib()
    table = np.array([L.orc_e2m1_decode(i) for i in range(16)], dtype=np.float64)
    return table[np.asarray(c, dtype=np.uint8) & 15]


def int8_encode(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.int8)
    lib().orc_int8_encode_n(_ptr(v), _ptr(out), v.size)
    return out


def mx_exponent(amax: np.ndarray) -> np.ndarray:
    amax = np.ascontiguousarray(amax, dtype=np.float32)
    out = np.empty(amax.shape, np.int32)
    lib().orc_mx_exponent_n(_ptr(amax), _ptr(out), amax.size)
    return out


def mx_exponent_e4m3(amax: np.ndarray) -> np.ndarray:
    amax = np.ascontiguousarray(amax, dtype=np.float32)
    out = np.empty(amax.shape, np.int32)
    lib().orc_mx_exponent_e4m3_n(_ptr(amax), _ptr(out), amax.size)
    return out


def f64_to_bf16(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, np.uint16)
    lib().orc_f64_to_bf16_n(_ptr(v), _ptr(out), v.size)
    return out


# ------------------------------------------------------------ quantizers ---

def calibrate_per_head(x: np.ndarray, layout: str = "BNSD",
                       amax: Optional[np.ndarray] = None) -> np.ndarray:
    """Running per-head max |x|; pass the previous result as ``amax`` to extend it."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    B, H, S, D = dims(x.shape, layout)
    a = np.zeros(H, np.float32) if amax is None else np.array(amax, dtype=np.float32, copy=True)
    lib().orc_calibrate_per_head(_ptr(x), B, H, S, D, LAYOUTS[layout], _ptr(a))
    return a


def quantize_int8_per_head(x: np.ndarray, amax: np.ndarray, layout: str = "BNSD"):
    x = np.ascontiguousarray(x, dtype=np.uint16)
    B, H, S, D = dims(x.shape, layout)
    amax = np.ascontiguousarray(amax, dtype=np.float32)
    codes = np.empty(x.shape, np.int8)
    scales = np.empty(H, np.float32)
    lib().orc_quantize_int8_per_head(_ptr(x), B, H, S, D, LAYOUTS[layout], _ptr(amax),
                                     _ptr(codes), _ptr(scales))
    return codes, scales


def quantize_fp8_per_token(x: np.ndarray, layout: str = "BNSD"):
    x = np.ascontiguousarray(x, dtype=np.uint16)
    B, H, S, D = dims(x.shape, layout)
    codes = np.empty(x.shape, np.uint8)
    scales = np.empty((B, H, S), np.float32)
    lib().orc_quantize_fp8_per_token(_ptr(x), B, H, S, D, LAYOUTS[layout], _ptr(codes), _ptr(scales))
    return codes, scales


def quantize_fp8_per_head(x: np.ndarray, amax: np.ndarray, layout: str = "BNSD"):
    x = np.ascontiguousarray(x, dtype=np.uint16)
    B, H, S, D = dims(x.shape, layout)
    amax = np.ascontiguousarray(amax, dtype=np.float32)
    codes = np.empty(x.shape, np.uint8)
    scales = np.empty(H, np.float32)
    lib().orc_quantize_fp8_per_head(_ptr(x), B, H, S, D, LAYOUTS[layout], _ptr(amax), _ptr(codes), _ptr(scales))
    return codes, scales


def quantize_int8_per_token(x: np.ndarray, layout: str = "BNSD"):
    x = np.ascontiguousarray(x, dtype=np.uint16)
    B, H, S, D = dims(x.shape, layout)
    codes = np.empty(x.shape, np.int8)
    scales = np.empty((B, H, S), np.float32)
    lib().orc_quantize_int8_per_token(_ptr(x), B, H, S, D, LAYOUTS[layout], _ptr(codes), _ptr(scales))
    return codes, scales


def quantize_mxfp4(x: np.ndarray, layout: str = "BNSD"):
    x = np.ascontiguousarray(x, dtype=np.uint16)
    B, H, S, D = dims(x.shape, layout)
    codes = np.empty(x.shape[:-1] + (D // 2,), np.uint8)
    e8m0 = np.empty((B, H, S, D // 32), np.uint8)
    lib().orc_quantize_mxfp4(_ptr(x), B, H, S, D, LAYOUTS[layout], _ptr(codes), _ptr(e8m0))
    return codes, e8m0


def quantize_mxfp8(x: np.ndarray, layout: str = "BNSD"):
    x = np.ascontiguousarray(x, dtype=np.uint16)
    B, H, S, D = dims(x.shape, layout)
    codes = np.empty(x.shape, np.uint8)
    e8m0 = np.empty((B, H, S, D // 32), np.uint8)
    lib().orc_quantize_mxfp8(_ptr(x), B, H, S, D, LAYOUTS[layout], _ptr(codes), _ptr(e8m0))
    return codes, e8m0


def rotate_f64(x: np.ndarray, R: np.ndarray, layout: str = "BNSD") -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.uint16)
    R = np.ascontiguousarray(R, dtype=np.uint16)
    B, H, S, D = dims(x.shape, layout)
    out = np.empty(x.shape, np.float64)
    lib().orc_rotate_f64(_ptr(x), B, H, S, D, LAYOUTS[layout], _ptr(R), _ptr(out))
    return out


def rotate(x: np.ndarray, R: np.ndarray, layout: str = "BNSD") -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.uint16)
    R = np.ascontiguousarray(R, dtype=np.uint16)
    B, H, S, D = dims(x.shape, layout)
    out = np.empty(x.shape, np.uint16)
    lib().orc_rotate(_ptr(x), B, H, S, D, LAYOUTS[layout], _ptr(R), _ptr(out))
    return out


def quantize_fp8_block(x: np.ndarray, blk: int, layout: str = "BNSD"):
    x = np.ascontiguousarray(x, dtype=np.uint16)
    B, H, S, D = dims(x.shape, layout)
    nblk = (S + blk - 1) // blk
    codes = np.empty(x.shape, np.uint8)
    scales = np.empty((B, H, nblk), np.float32)
    lib().orc_quantize_fp8_block(_ptr(x), B, H, S, D, LAYOUTS[layout], blk, _ptr(codes), _ptr(scales))
    return codes, scales


# ------------------------------------------------- dequant and attention ---

@dataclass
class QT:
    """An operand as the oracle sees it (codes + scales + mode + layout)."""
    mode: str
    codes: np.ndarray
    scales: Optional[np.ndarray]
    B: int
    H: int
    S: int
    D: int
    layout: str = "BNSD"
    blk: int = 0

    def _c(self) -> _OrcQT:
        self._keep = (np.ascontiguousarray(self.codes),
                      None if self.scales is None else np.ascontiguousarray(self.scales))
        return _OrcQT(MODES[self.mode], self._keep[0].ctypes.data,
                      0 if self._keep[1] is None else self._keep[1].ctypes.data,
                      self.B, self.H, self.S, self.D, LAYOUTS[self.layout], self.blk)


def qt_float(x: np.ndarray, layout: str = "BNSD") -> QT:
    B, H, S, D = dims(x.shape, layout)
    return QT("float", np.ascontiguousarray(x, dtype=np.uint16), None, B, H, S, D, layout)


def dequant_head(t: QT, b: int, h: int) -> np.ndarray:
    out = np.empty((t.S, t.D), np.float64)
    c = t._c()
    lib().orc_dequant_head(ctypes.byref(c), b, h, _ptr(out))
    return out


def dequant(t: QT) -> np.ndarray:
    """Full dequantized tensor, canonical [B, H, S, D] fp64."""
    out = np.empty((t.B, t.H, t.S, t.D), np.float64)
    for b in range(t.B):
        for h in range(t.H):
            out[b, h] = dequant_head(t, b, h)
    return out


def attention(q: QT, k: QT, v: QT, causal: bool = False, scale: float = 0.0,
              rows: Optional[Sequence[int]] = None):
    """Exact fp64 attention on the dequantized operands.

    Returns (out [B, Hq, nrows, D] fp64, lse [B, Hq, nrows] fp64)."""
    if rows is None:
        rows_arr, nrows, rp = None, q.S, 0
    else:
        rows_arr = np.ascontiguousarray(rows, dtype=np.int32)
        nrows, rp = rows_arr.size, rows_arr.ctypes.data
    out = np.empty((q.B, q.H, nrows, q.D), np.float64)
    lse = np.empty((q.B, q.H, nrows), np.float64)
    cq, ck, cv = q._c(), k._c(), v._c()
    lib().orc_attention(ctypes.byref(cq), ctypes.byref(ck), ctypes.byref(cv), int(bool(causal)),
                        float(scale), rp, nrows, _ptr(out), _ptr(lse))
    return out, lse
