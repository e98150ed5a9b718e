"""Python binding of the FA-quantization C ABI (include/faq.h).

Argument marshalling only: every step of the path runs in libfaq.so's CUDA
kernels.  PyTorch supplies device memory and the current CUDA stream.
Tensors are bf16 CUDA tensors shaped [B, H, S, D] (layout "BNSD") or
[B, S, H, D] (layout "BSND").
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional, Sequence, Tuple

import torch

from . import _native as N

LAYOUTS = {"BNSD": 0, "BSND": 1}
MODES = {"float": 0, "int8_per_head": 1, "fp8_per_token": 2, "mxfp4": 3, "fp8_block": 4, "fp8_per_head": 5,
         "int8_per_token": 6, "mxfp8": 7}
MODE_NAMES = {v: k for k, v in MODES.items()}


class FaqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {N.STATUS.get(status, status)} ({N.lib().fa_status_str(status).decode()})")


def _check(st: int, where: str):
    if st != 0:
        raise FaqError(st, where)


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def dims(shape: Sequence[int], layout: str) -> Tuple[int, int, int, int]:
    if layout == "BNSD":
        B, H, S, D = shape
    elif layout == "BSND":
        B, S, H, D = shape
    else:
        raise ValueError(f"layout must be BNSD or BSND, got {layout!r}")
    return B, H, S, D


def _shape(B, H, S, D, layout):
    return (B, H, S, D) if layout == "BNSD" else (B, S, H, D)


@dataclass
class QTensor:
    """Codes + scales + mode + layout (fa_qtensor)."""
    codes: torch.Tensor
    scales: torch.Tensor
    mode: str
    B: int
    H: int
    S: int
    D: int
    layout: str = "BNSD"
    block_tokens: int = 0

    def c(self) -> N.FaQTensor:
        return N.FaQTensor(self.codes.data_ptr(), self.scales.data_ptr() if self.scales is not None else None,
                           MODES[self.mode], self.B, self.H, self.S, self.D, LAYOUTS[self.layout],
                           self.block_tokens)


def float_branch(x: torch.Tensor, layout: str = "BNSD") -> QTensor:
    """An unquantized branch for attention (FA_MODE_FLOAT): the bf16 tensor itself."""
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("expected a contiguous bf16 CUDA tensor")
    B, H, S, D = dims(x.shape, layout)
    return QTensor(x, None, "float", B, H, S, D, layout)


def empty_qtensor(B: int, H: int, S: int, D: int, mode: str, layout: str = "BNSD", block_tokens: int = 0,
                  device="cuda") -> QTensor:
    """Allocate (with torch) the code and scale buffers for one operand."""
    shp = _shape(B, H, S, D, layout)
    if mode == "int8_per_head":
        codes = torch.empty(shp, dtype=torch.int8, device=device)
        scales = torch.empty((H,), dtype=torch.float32, device=device)
    elif mode == "fp8_per_head":
        codes = torch.empty(shp, dtype=torch.uint8, device=device)
        scales = torch.empty((H,), dtype=torch.float32, device=device)
    elif mode == "int8_per_token":
        codes = torch.empty(shp, dtype=torch.int8, device=device)
        scales = torch.empty((B, H, S), dtype=torch.float32, device=device)
    elif mode == "fp8_per_token":
        codes = torch.empty(shp, dtype=torch.uint8, device=device)
        scales = torch.empty((B, H, S), dtype=torch.float32, device=device)
    elif mode == "fp8_block":
        if block_tokens < 1:
            raise ValueError("fp8_block needs block_tokens >= 1")
        codes = torch.empty(shp, dtype=torch.uint8, device=device)
        scales = torch.empty((B, H, (S + block_tokens - 1) // block_tokens), dtype=torch.float32, device=device)
    elif mode == "mxfp4":
        codes = torch.empty(shp[:-1] + (D // 2,), dtype=torch.uint8, device=device)
        scales = torch.empty((B, H, S, D // 32), dtype=torch.uint8, device=device)
    elif mode == "mxfp8":
        codes = torch.empty(shp, dtype=torch.uint8, device=device)
        scales = torch.empty((B, H, S, D // 32), dtype=torch.uint8, device=device)
    else:
        raise ValueError(f"unknown mode {mode!r}")
    return QTensor(codes, scales, mode, B, H, S, D, layout, block_tokens)


def _tensor(x: torch.Tensor, layout: str) -> N.FaTensor:
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("expected a contiguous bf16 CUDA tensor")
    B, H, S, D = dims(x.shape, layout)
    return N.FaTensor(x.data_ptr(), B, H, S, D, LAYOUTS[layout])


def resolve_config(qconfig: Optional[str] = None, details: Optional[Sequence[Optional[str]]] = None):
    """Branch modes (q, k, v) from a unified qconfig or per-branch details
    (fa_resolve_config).  Host only."""
    q = N.FaBranchCfg(1, MODES[qconfig]) if qconfig is not None else None
    d = None
    if details is not None:
        arr = (N.FaBranchCfg * 3)()
        for i, m in enumerate(details):
            arr[i] = N.FaBranchCfg(0, 0) if m is None else N.FaBranchCfg(1, MODES[m])
        d = arr
    out = (ctypes.c_int * 3)()
    _check(N.lib().fa_resolve_config(ctypes.byref(q) if q is not None else None, d, out), "fa_resolve_config")
    return tuple(MODE_NAMES[out[i]] for i in range(3))


def calibrate_per_head(x: torch.Tensor, layout: str = "BNSD", amax: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Running per-head max |x| (fa_calibrate_per_head).  Pass the previous
    result as ``amax`` to fold in another batch."""
    t = _tensor(x, layout)
    if amax is None:
        amax = torch.zeros(t.H, dtype=torch.float32, device=x.device)
    _check(N.lib().fa_calibrate_per_head(ctypes.byref(t), amax.data_ptr(), _stream()), "fa_calibrate_per_head")
    return amax


def quantize(q: Optional[torch.Tensor], k: Optional[torch.Tensor], v: Optional[torch.Tensor], mode: str,
             layout: str = "BNSD", amax: Optional[Sequence[Optional[torch.Tensor]]] = None, q_block: int = 128,
             kv_block: int = 256, out: Optional[Sequence[Optional[QTensor]]] = None):
    """Quantize Q, K, V with one unified mode in one launch (fa_quantize).
    Returns a tuple of QTensor (None for an operand passed as None)."""
    ins = (q, k, v)
    am = tuple(amax) if amax is not None else (None, None, None)
    blks = (q_block, kv_block, kv_block)
    ts, outs = [], []
    for i, x in enumerate(ins):
        if x is None:
            ts.append(None)
            outs.append(None)
            continue
        t = _tensor(x, layout)
        ts.append(t)
        o = out[i] if out is not None and out[i] is not None else empty_qtensor(
            t.B, t.H, t.S, t.D, mode, layout, blks[i] if mode == "fp8_block" else 0, x.device)
        outs.append(o)
    cq = [o.c() if o is not None else None for o in outs]
    refs = [ctypes.byref(t) if t is not None else None for t in ts]
    orefs = [ctypes.byref(c) if c is not None else None for c in cq]
    amp = [a.data_ptr() if a is not None else None for a in am]
    _check(N.lib().fa_quantize(refs[0], refs[1], refs[2], MODES[mode], amp[0], amp[1], amp[2],
                               orefs[0], orefs[1], orefs[2], _stream()), "fa_quantize")
    return tuple(outs)


def rotate_quantize(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, rot_q: torch.Tensor, rot_k: torch.Tensor,
                    layout: str = "BNSD", q_block: int = 128, kv_block: int = 256, debug: bool = False,
                    out: Optional[Sequence[QTensor]] = None):
    """Rotate Q and K, then FP8 block-quantize Q, K, V (fa_rotate_quantize).
    Returns (Qq, Kq, Vq) or, with debug=True, (Qq, Kq, Vq, Q_rot, K_rot).
    ``out`` reuses existing output QTensors (e.g. inside a CUDA graph)."""
    ts = [_tensor(x, layout) for x in (q, k, v)]
    blks = (q_block, kv_block, kv_block)
    outs = list(out) if out is not None else [
        empty_qtensor(t.B, t.H, t.S, t.D, "fp8_block", layout, blks[i], q.device) for i, t in enumerate(ts)]
    for R in (rot_q, rot_k):
        if R.dtype != torch.bfloat16 or not R.is_cuda or not R.is_contiguous() or R.shape != (ts[0].D, ts[0].D):
            raise ValueError("rotation must be a contiguous bf16 CUDA tensor [D, D]")
    dq = torch.empty_like(q) if debug else None
    dk = torch.empty_like(k) if debug else None
    cq = [o.c() for o in outs]
    _check(N.lib().fa_rotate_quantize(ctypes.byref(ts[0]), ctypes.byref(ts[1]), ctypes.byref(ts[2]),
                                      rot_q.data_ptr(), rot_k.data_ptr(), q_block, kv_block,
                                      ctypes.byref(cq[0]), ctypes.byref(cq[1]), ctypes.byref(cq[2]),
                                      dq.data_ptr() if dq is not None else None,
                                      dk.data_ptr() if dk is not None else None, _stream()),
           "fa_rotate_quantize")
    return tuple(outs) + ((dq, dk) if debug else ())


def rotate_quantize_hadamard(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, signs_q, signs_k,
                             layout: str = "BNSD", q_block: int = 128, kv_block: int = 256, debug: bool = False,
                             out: Optional[Sequence[QTensor]] = None):
    """Rotate Q and K by R = bf16(H_D diag(signs) / sqrt(D)), given by its signs, then FP8
    block-quantize Q, K, V (fa_rotate_quantize_hadamard: R built on chip for D = 128 with blocks
    dividing 256, a fast Walsh-Hadamard transform otherwise).  signs_q / signs_k: sequences of D
    values +1 / -1 (or None for all +1).  Returns as rotate_quantize."""
    ts = [_tensor(x, layout) for x in (q, k, v)]
    D = ts[0].D
    blks = (q_block, kv_block, kv_block)
    outs = list(out) if out is not None else [
        empty_qtensor(t.B, t.H, t.S, t.D, "fp8_block", layout, blks[i], q.device) for i, t in enumerate(ts)]

    def bits(signs):
        if signs is None:
            return None
        sg = [int(x) for x in signs]
        if len(sg) != D or any(x not in (1, -1) for x in sg):
            raise ValueError(f"signs must be {D} values of +1 / -1")
        words = (ctypes.c_uint32 * (D // 32))()
        for j, x in enumerate(sg):
            if x < 0:
                words[j // 32] |= 1 << (j % 32)
        return words

    bq, bk = bits(signs_q), bits(signs_k)
    dq = torch.empty_like(q) if debug else None
    dk = torch.empty_like(k) if debug else None
    cq = [o.c() for o in outs]
    _check(N.lib().fa_rotate_quantize_hadamard(ctypes.byref(ts[0]), ctypes.byref(ts[1]), ctypes.byref(ts[2]),
                                               bq, bk, q_block, kv_block,
                                               ctypes.byref(cq[0]), ctypes.byref(cq[1]), ctypes.byref(cq[2]),
                                               dq.data_ptr() if dq is not None else None,
                                               dk.data_ptr() if dk is not None else None, _stream()),
           "fa_rotate_quantize_hadamard")
    return tuple(outs) + ((dq, dk) if debug else ())


def attention_workspace_size(q: QTensor, k: QTensor, num_splits: int = 0, v: Optional[QTensor] = None) -> int:
    cq, ck = q.c(), k.c()
    if v is not None:
        cv = v.c()
        return int(N.lib().fa_attention_workspace_size_qkv(ctypes.byref(cq), ctypes.byref(ck), ctypes.byref(cv),
                                                           num_splits))
    return int(N.lib().fa_attention_workspace_size(ctypes.byref(cq), ctypes.byref(ck), num_splits))


def attention(q: QTensor, k: QTensor, v: QTensor, causal: bool = False, softmax_scale: float = 0.0,
              out: Optional[torch.Tensor] = None, return_lse: bool = False, num_splits: int = 0,
              workspace: Optional[torch.Tensor] = None):
    """Attention on quantized operands, bf16 output in q's layout
    (fa_attention_quant).  Each branch may have its own mode; ``float_branch``
    wraps an unquantized one.  Returns out, or (out, lse) with return_lse."""
    dev = q.codes.device
    if out is None:
        out = torch.empty(_shape(q.B, q.H, q.S, q.D, q.layout), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((q.B, q.H, q.S), dtype=torch.float32, device=dev) if return_lse else None
    cq, ck, cv = q.c(), k.c(), v.c()
    need = int(N.lib().fa_attention_workspace_size_qkv(ctypes.byref(cq), ctypes.byref(ck), ctypes.byref(cv),
                                                       num_splits))
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(N.lib().fa_attention_quant(ctypes.byref(cq), ctypes.byref(ck), ctypes.byref(cv), int(bool(causal)),
                                      float(softmax_scale), out.data_ptr(),
                                      lse.data_ptr() if lse is not None else None, int(num_splits), ws_ptr,
                                      ws_bytes, _stream()), "fa_attention_quant")
    return (out, lse) if return_lse else out


def decode_append(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, amax: Sequence[torch.Tensor],
                  k_cache: QTensor, v_cache: QTensor, pos: int, softmax_scale: float = 0.0,
                  out: Optional[torch.Tensor] = None, return_lse: bool = False, num_splits: int = 0,
                  workspace: Optional[torch.Tensor] = None):
    """One decode step on an INT8 per-head cache (fa_decode_append): q, k_new, v_new are the new
    token's bf16 rows ([B, H, 1, D] in the cache's layout); k_new / v_new are quantized into the
    caches at ``pos``, then attention runs over the first pos + 1 cached tokens.  ``amax`` holds
    the per-head calibration maxima for q, k, v.  Returns out, or (out, lse)."""
    layout = k_cache.layout
    tq, tk, tv = _tensor(q, layout), _tensor(k_new, layout), _tensor(v_new, layout)
    dev = q.device
    if out is None:
        out = torch.empty(_shape(tq.B, tq.H, 1, tq.D, layout), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((tq.B, tq.H, 1), dtype=torch.float32, device=dev) if return_lse else None
    ck, cv = k_cache.c(), v_cache.c()
    need = int(N.lib().fa_decode_append_workspace_size(ctypes.byref(tq), ctypes.byref(ck), int(pos), num_splits))
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(N.lib().fa_decode_append(ctypes.byref(tq), ctypes.byref(tk), ctypes.byref(tv), amax[0].data_ptr(),
                                    amax[1].data_ptr(), amax[2].data_ptr(), ctypes.byref(ck), ctypes.byref(cv),
                                    int(pos), float(softmax_scale), out.data_ptr(),
                                    lse.data_ptr() if lse is not None else None, int(num_splits),
                                    workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream()),
           "fa_decode_append")
    return (out, lse) if return_lse else out


def check_device_status():
    """Synchronise the current stream and raise if a kernel's bounded wait ran out."""
    _check(N.lib().fa_check_device_status(_stream()), "fa_check_device_status")


def version() -> str:
    return N.lib().fa_version().decode()
