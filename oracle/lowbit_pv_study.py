"""Numerical study behind a design decision (test infrastructure, CPU only): P·V with both operands
in E4M3 against the exact attention, on the full-size workloads' quantized operands.

    python -m oracle.lowbit_pv_study [--rows 64] [--heads 4] [--psh 8] [--workloads ...]

Reading studied (MindIE SD "量化", FA量化 / 技术特点, FP8 Attention: the attention runs in the FP8
domain): per 128-key tile t, V' = e4m3(V^ / 2^e_t) with the power-of-two tile scale 2^e_t that
puts max |V^_t| at or under 448; P' = e4m3(p * 2^(e_t - e_ref)) with p = exp(s - m) (m the row's
final maximum, the most favourable case for P) and e_ref = max_t e_t, times 2^psh (headroom that
keeps small weights in E4M3's normal range); the row sum l taken from the quantized P' (the
rounded weights then still sum to one); O = 2^e_ref * sum P' V' / l.  A second form, for V with
one E4M3 scale per key (per token or per block): V' = the codes themselves (exact), each key's
scale folded into P' = e4m3(p * s_j / s_ref * 2^psh).  The exact side is the oracle's fp64
attention on the same dequantized operands.
Printed per workload: the largest max-abs error per row and its mean, both divided by M_h (the
largest |V^| of the head), over the sampled rows and heads -- the quantities the attention
tolerance (2e-2 and 2e-3 of M_h) bounds.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
if os.path.dirname(HERE) not in sys.path:
    sys.path.insert(0, os.path.dirname(HERE))

import oracle as orc  # noqa: E402
import workloads as wl  # noqa: E402

TILE = 128
PSH = 8  # power-of-two headroom of P' (2^8 * p <= 256 < 448): small weights stay normal E4M3


def quantize_operand(w, name, x):
    bits = wl.bf16_bits(x)
    if w.mode == "fp8_per_token":
        c, s = orc.quantize_fp8_per_token(bits, w.layout)
        blk = 0
    elif w.mode == "fp8_block":
        blk = w.q_block if name == "q" else w.kv_block
        c, s = orc.quantize_fp8_block(bits, blk, w.layout)
    elif w.mode == "mxfp4":
        c, s = orc.quantize_mxfp4(bits, w.layout)
        blk = 0
    else:
        raise ValueError(w.mode)
    B, H, S, D = orc.dims(bits.shape, w.layout)
    return orc.QT(w.mode, c, s, B, H, S, D, w.layout, blk)


def e4m3(v: np.ndarray) -> np.ndarray:
    return orc.e4m3_decode(orc.e4m3_encode(v.astype(np.float32)))


def study(name: str, nrows: int, nheads: int, seed: int = 0):
    w = wl.WORKLOADS[name]
    inp = wl.make_inputs(w, calib=False)
    q, k, v = inp["q"], inp["k"], inp["v"]
    if w.rotate:
        Rb = wl.bf16_bits(inp["R"])
        qb = orc.rotate(wl.bf16_bits(q), Rb, w.layout)
        kb = orc.rotate(wl.bf16_bits(k), Rb, w.layout)
        Q = _qt_from_bits(w, "q", qb)
        K = _qt_from_bits(w, "k", kb)
    else:
        Q = quantize_operand(w, "q", q)
        K = quantize_operand(w, "k", k)
    V = quantize_operand(w, "v", v)
    rng = np.random.default_rng(seed)
    group = w.Hq // w.Hkv
    heads = sorted(rng.choice(w.Hq, size=min(nheads, w.Hq), replace=False).tolist())
    fixed = [r for r in list(range(0, 40)) + [127, 128, 255, 256, w.Sq - 1] if r < w.Sq]
    rows = sorted(set(fixed + rng.choice(w.Sq, size=max(0, nrows - len(fixed)), replace=False).tolist()))
    diag = w.Sk - w.Sq
    worst_max, worst_mean, worst_max_l, fold_max, fold_mean, fold_late = 0.0, 0.0, 0.0, 0.0, 0.0, 0.0
    for b in range(w.B):
        for h in heads:
            hk = h // group
            qh = orc.dequant_head(Q, b, h)
            kh = orc.dequant_head(K, b, hk)
            vh = orc.dequant_head(V, b, hk)
            M = np.abs(vh).max()
            nt = -(-w.Sk // TILE)
            # V' per tile with a power-of-two scale: max |V^_t| / 2^e_t <= 448
            e = np.zeros(nt)
            vq = np.empty_like(vh)
            for t in range(nt):
                vt = vh[t * TILE:(t + 1) * TILE]
                mt = np.abs(vt).max()
                e[t] = np.ceil(np.log2(mt / 448.0)) if mt > 0 else 0.0
                vq[t * TILE:(t + 1) * TILE] = e4m3(vt / 2.0 ** e[t])
            errs, means, errs_l, errs_f, means_f, late_f = [], [], [], [], [], []
            vcodes, vscale = per_key_codes(V, b, hk)
            for r in rows:
                last = min(w.Sk - 1, r + diag) if w.causal else w.Sk - 1
                if last < 0:
                    continue
                s = kh[:last + 1] @ qh[r] / np.sqrt(w.D)
                p = np.exp(s - s.max())
                o = p @ vh[:last + 1] / p.sum()
                et = e[np.arange(last + 1) // TILE]
                eref = et.max()
                fold = 2.0 ** (et - eref)
                # P' scaled by 2^PSH so that small weights stay in E4M3's normal range (<= 256 < 448)
                pq = e4m3(p * fold * 2.0 ** PSH)
                l_q = (pq / fold).sum()
                o_low = 2.0 ** eref * (pq @ vq[:last + 1]) / l_q
                o_low_l = 2.0 ** (eref - PSH) * (pq @ vq[:last + 1]) / p.sum()  # l from the unquantized p
                if vcodes is not None:
                    # variant: V' = the E4M3 codes themselves (exact), each key's V scale folded into P'
                    sv = vscale[:last + 1]
                    sref = sv.max()
                    fk = sv / sref
                    pk = e4m3(p * fk * 2.0 ** PSH)
                    o_fold = sref * (pk @ vcodes[:last + 1]) / (pk / fk).sum()
                    errs_f.append(np.abs(o_fold - o).max() / M)
                    if r >= TILE:
                        late_f.append(errs_f[-1])
                    means_f.append(np.abs(o_fold - o).mean() / M)
                errs.append(np.abs(o_low - o).max() / M)
                means.append(np.abs(o_low - o).mean() / M)
                errs_l.append(np.abs(o_low_l - o).max() / M)
            worst_max = max(worst_max, max(errs))
            worst_mean = max(worst_mean, float(np.mean(means)))
            worst_max_l = max(worst_max_l, max(errs_l))
            if late_f:
                fold_late = max(fold_late, max(late_f))
            if errs_f:
                fold_max = max(fold_max, max(errs_f))
                fold_mean = max(fold_mean, float(np.mean(means_f)))
    print(f"{name:14s} rows {len(rows):4d} x heads {len(heads)} x batches {w.B}:  "
          f"max err {worst_max:.4f} M_h, mean err {worst_mean:.5f} M_h  "
          f"(l from unquantized p: max {worst_max_l:.4f} M_h)" +
          (f"; V scale folded into P', V' = codes: max {fold_max:.4f} M_h, mean {fold_mean:.5f} M_h, "
           f"rows >= {TILE}: max {fold_late:.4f} M_h" if fold_max > 0 else ""), flush=True)
    return worst_max, worst_mean


def per_key_codes(V, b, hk):
    """For E4M3 V with one scale per key (per token, or per block of tokens): the decoded codes
    [S, D] and each key's scale [S]; (None, None) for other modes."""
    if V.mode not in ("fp8_per_token", "fp8_block"):
        return None, None
    if V.layout == "BNSD":
        codes = V.codes[b, hk]
    else:
        codes = V.codes[b, :, hk]
    vals = orc.e4m3_decode(np.ascontiguousarray(codes).reshape(-1)).reshape(codes.shape)
    if V.mode == "fp8_per_token":
        sc = np.asarray(V.scales[b, hk], np.float64)
    else:
        sc = np.repeat(np.asarray(V.scales[b, hk], np.float64), V.blk)[:V.S]
    return vals, sc


def _qt_from_bits(w, name, bits):
    blk = w.q_block if name == "q" else w.kv_block
    c, s = orc.quantize_fp8_block(bits, blk, w.layout)
    B, H, S, D = orc.dims(bits.shape, w.layout)
    return orc.QT(w.mode, c, s, B, H, S, D, w.layout, blk)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--rows", type=int, default=64)
    ap.add_argument("--heads", type=int, default=4)
    ap.add_argument("--workloads", default="fp8_prefill,rot_fp8_block,mxfp4")
    ap.add_argument("--psh", type=int, default=PSH, help="P' headroom: P' = e4m3(p * fold * 2^psh)")
    a = ap.parse_args()
    globals()["PSH"] = a.psh
    for name in a.workloads.split(","):
        study(name, a.rows, a.heads)


if __name__ == "__main__":
    main()
