#!/usr/bin/env python
"""bench.py -- throughput of the FA-quantization hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl faq|reference]
                    [--workload NAME] [--no-supplemental]

One step is one pass of the whole hot path over one batch of synthetic,
seeded input already resident in HBM: quantize Q/K/V (or rotate + block
quantize), then attention on the low-bit operands.  The default workload is
the FP8 E4M3 per-token LLM prefill (B=2, Hq=32, Hkv=8, S=4096, D=128,
causal, GQA, BNSD); --workload picks another (int8_tiny, rot_fp8_block,
mxfp4, int8_decode).  Each step is a CUDA-graph replay timed with CUDA
events on its stream, with L2 flushed between steps (a 256 MiB write, then a
256 MiB read so that no dirty line of the flush is left for the timed kernels
to write back).
Prints one JSON line (rank 0).  Under torchrun every rank runs its own
independent replica of the workload (weak scaling, no data-path collective);
time is the max over ranks.

--impl reference times the oracle (the CPU statement of the method) on the
box's host cores, each step a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quant-attn TFLOP/s & % of FP8/INT8/FP4 dense peak; decode KV GB/s vs 8 TB/s"
L2_FLUSH_BYTES = 256 << 20

DESCR = {
    "int8_tiny": "INT8 per-head static, B=1 H=2 S=256 D=64, non-causal, BNSD",
    "fp8_prefill": "FP8 E4M3 per-token dynamic, LLM prefill, B=2 Hq=32 Hkv=8 S=4096 D=128, causal, BNSD",
    "rot_fp8_block": "rotate -> FP8 block quant (Q 128 / KV 256 tokens), video-DiT B=1 H=40 S=32768 D=128, "
                     "non-causal, BSND",
    "mxfp4": "MXFP4 per-32-block (E2M1 + E8M0), image-edit B=1 H=24 S=4096 D=128, non-causal, BNSD, Student-t",
    "int8_decode": "INT8 per-head static split-KV decode, B=16 Hq=32 Hkv=8 Sq=1 Sk=32768 D=128, BNSD",
    "int8_prefill": "INT8 per-head static, the fp8_prefill shape (B=2 Hq=32 Hkv=8 S=4096 D=128, causal, BNSD)",
    "fp8_head_prefill": "FP8 E4M3 per-head static, the fp8_prefill shape (B=2 Hq=32 Hkv=8 S=4096 D=128, causal, BNSD)",
    "int8_token_prefill": "INT8 per-token dynamic, the fp8_prefill shape (B=2 Hq=32 Hkv=8 S=4096 D=128, causal, BNSD)",
    "mxfp8": "MXFP8 per-32-block (E4M3 + E8M0), the mxfp4 shape (B=1 H=24 S=4096 D=128, non-causal, BNSD, Student-t)",
    "mixed_prefill": "per-branch modes: Q, K FP8 per-token, V unquantized bf16, the fp8_prefill shape "
                     "(B=2 Hq=32 Hkv=8 S=4096 D=128, causal, BNSD)",
}
DATA = {
    "int8_tiny": "synthetic: seeded bf16 N(0,1); per-head scales from a seeded calibration batch",
    "fp8_prefill": "synthetic: seeded bf16 N(0,1); K with 4 seeded head_dim channels per kv head x20",
    "rot_fp8_block": "synthetic: seeded bf16 N(0,1); R = bf16(Hadamard * seeded signs / sqrt(128))",
    "mxfp4": "synthetic: seeded bf16 Student-t (df=4)",
    "int8_decode": "synthetic: seeded bf16 N(0,1) cache and query; per-head scales from seeded calibration batches",
    "int8_prefill": "synthetic: as fp8_prefill; per-head scales from seeded calibration batches",
    "fp8_head_prefill": "synthetic: as fp8_prefill; per-head scales from seeded calibration batches",
    "int8_token_prefill": "synthetic: as fp8_prefill",
    "mxfp8": "synthetic: seeded bf16 Student-t (df=4)",
    "mixed_prefill": "synthetic: as fp8_prefill",
}
DTYPE = {
    "int8_tiny": "s8 (QK^T, s32 acc) + f16 (PV)",
    "fp8_prefill": "e4m3 (QK^T) + f16 (PV), fp32 accumulate",
    "rot_fp8_block": "bf16 (rotation) + e4m3 (QK^T) + f16 (PV)",
    "mxfp4": "e2m1 block-scaled (QK^T) + f16 (PV)",
    "int8_decode": "s8 (QK^T) + u8/s8 (PV), s32 accumulate",
    "int8_prefill": "s8 (QK^T, s32 acc) + f16 (PV)",
    "fp8_head_prefill": "e4m3 (QK^T) + f16 (PV), fp32 accumulate",
    "int8_token_prefill": "s8 (QK^T, s32 acc) + f16 (PV)",
    "mxfp8": "e4m3 block-scaled (QK^T) + f16 (PV)",
    "mixed_prefill": "bf16 (dequantized QK^T) + f16 (PV), fp32 accumulate",
}


# modes whose scales come from a calibration batch (per-head static)
STATIC_MODES = ("int8_per_head", "fp8_per_head")

def attn_flops(w) -> float:
    """Algorithmic attention FLOPs: 4 * D per unmasked (query, key) pair."""
    if w.causal:
        diag = w.Sk - w.Sq
        pairs = sum(max(0, min(w.Sk, i + diag + 1)) for i in range(w.Sq))
    else:
        pairs = w.Sq * w.Sk
    return 4.0 * w.B * w.Hq * w.D * pairs


def quant_bytes(w) -> float:
    """Algorithmic bytes of the quantize step: bf16 in once, codes + scales out once."""
    nq = w.B * w.Hq * w.Sq * w.D
    nk = w.B * w.Hkv * w.Sk * w.D
    if w.branch_modes is not None:
        # this bench's mixed workload: Q and K FP8 per token, V not quantized
        assert w.branch_modes == ("fp8_per_token", "fp8_per_token", "float")
        return (nq + nk) * 3 + (w.B * w.Hq * w.Sq + w.B * w.Hkv * w.Sk) * 4
    if w.mode == "int8_decode" or w.name == "int8_decode":
        return nq * 2 + nq + w.Hq * 4  # only Q is quantized per step
    code = 0.5 if w.mode == "mxfp4" else 1.0
    if w.mode in ("fp8_per_token", "int8_per_token"):
        sc = (w.B * w.Hq * w.Sq + 2 * w.B * w.Hkv * w.Sk) * 4
    elif w.mode == "fp8_block":
        sc = (w.B * w.Hq * -(-w.Sq // w.q_block) + 2 * w.B * w.Hkv * -(-w.Sk // w.kv_block)) * 4
    elif w.mode in ("mxfp4", "mxfp8"):
        sc = (nq + 2 * nk) // 32
    else:
        sc = (w.Hq + 2 * w.Hkv) * 4
    return (nq + 2 * nk) * (2 + code) + sc


def decode_bytes(w) -> float:
    """Algorithmic bytes of split-KV decode: K and V codes once + Q codes + bf16 output."""
    return 2.0 * w.B * w.Hkv * w.Sk * w.D + w.B * w.Hq * w.D * (1 + 2)


def peaks():
    p = {}
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        try:
            p = json.load(open(path))
        except Exception:
            p = {}
    if "hbm_gbs" in p and "bf16_tflops" in p:
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16": float(p["bf16_tflops"]),
                "bf16_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "src": "fallback"}


def tensor_peak(w, pk):
    """Dense peak for the QK^T operand type: measured bf16 x the nominal ratio
    (FP8/INT8 2x, FP4 4x the bf16 rate; bf16 itself for mixed branches)."""
    ratio = 4.0 if w.mode == "mxfp4" else 2.0
    if w.branch_modes is not None:
        ratio = 1.0  # mixed branches: QK^T on bf16
    return pk["bf16"] * ratio


# ---------------------------------------------------------------- clocks ---

class ClockSampler:
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid=None):
        self.uuid = uuid
        self.proc = None
        self.path = os.path.join("/tmp", f"faq_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            if self.uuid and parts[1] != self.uuid:
                continue
            rows.append(parts)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[6:10]) if v.lower() == "active"})
        under = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(under) if under else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------- GPU arm ---

ROTATION = "matrix"  # rotating workloads: fa_rotate_quantize with R, or fa_rotate_quantize_hadamard


def make_step(faq, wl, w, device, seed_offset=0):
    """Allocate inputs on the device and return (step_fn, attn_fn, quant_fn, state)."""
    import torch
    w2 = w.scaled(seed=w.seed + seed_offset)
    inp = wl.make_inputs(w2, device=device, calib=(w.mode in STATIC_MODES))
    q, k, v = inp["q"], inp["k"], inp["v"]
    st = {"inp": inp}
    if w.mode in STATIC_MODES:
        amax = [faq.calibrate_per_head(inp[n + "_cal"], w.layout) for n in "qkv"]
        st["amax"] = amax
        if w.name == "int8_decode":
            # the K/V cache is quantized once, outside the step
            _, Kq, Vq = faq.quantize(None, k, v, w.mode, w.layout, amax=[None, amax[1], amax[2]])
            Qq = faq.quantize(q, None, None, w.mode, w.layout, amax=[amax[0], None, None])[0]
            qout = [Qq, None, None]
            st["QKV"] = [Qq, Kq, Vq]

            def quant():
                faq.quantize(q, None, None, w.mode, w.layout, amax=[amax[0], None, None], out=qout)
        else:
            QKV = list(faq.quantize(q, k, v, w.mode, w.layout, amax=amax))
            st["QKV"] = QKV

            def quant():
                faq.quantize(q, k, v, w.mode, w.layout, amax=amax, out=QKV)
    elif w.branch_modes is not None:
        # Q and K quantized in one mode, V left as bf16 (the only mix this bench runs)
        mq, mk, mv = w.branch_modes
        assert mq == mk and mv == "float"
        QK = list(faq.quantize(q, k, None, mq, w.layout))
        st["QKV"] = [QK[0], QK[1], faq.float_branch(v, w.layout)]

        def quant():
            faq.quantize(q, k, None, mq, w.layout, out=QK)
    elif w.rotate and ROTATION == "hadamard":
        # the same rotation given by its signs (R = bf16(H diag(signs) / sqrt(D)))
        sg = wl.rotation_signs(w.D, w2.seed)
        QKV = list(faq.rotate_quantize_hadamard(q, k, v, sg, sg, w.layout, w.q_block, w.kv_block))
        st["QKV"] = QKV

        def quant():
            faq.rotate_quantize_hadamard(q, k, v, sg, sg, w.layout, w.q_block, w.kv_block, out=QKV)
    elif w.rotate:
        QKV = list(faq.rotate_quantize(q, k, v, inp["R"], inp["R"], w.layout, w.q_block, w.kv_block))
        st["QKV"] = QKV

        def quant():
            faq.rotate_quantize(q, k, v, inp["R"], inp["R"], w.layout, w.q_block, w.kv_block, out=QKV)
    else:
        QKV = list(faq.quantize(q, k, v, w.mode, w.layout, q_block=w.q_block, kv_block=w.kv_block))
        st["QKV"] = QKV

        def quant():
            faq.quantize(q, k, v, w.mode, w.layout, q_block=w.q_block, kv_block=w.kv_block, out=QKV)

    Qq, Kq, Vq = st["QKV"]
    out = torch.empty_like(q)
    ws_bytes = faq.attention_workspace_size(Qq, Kq, v=Vq)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=device)
    st["out"] = out

    def attn():
        faq.attention(Qq, Kq, Vq, causal=w.causal, out=out, workspace=ws)

    def step():
        quant()
        attn()

    return step, attn, quant, st


class L2Flush:
    """Flush L2 between timed steps: write a buffer larger than L2 (126 MB), then read
    another one, so the next step starts with none of its inputs in L2 and without the
    write's dirty lines, which the timed kernels would otherwise write back to HBM."""

    def __init__(self, device):
        import torch
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
        self.sink = torch.empty((), dtype=torch.float32, device=device)

    def __call__(self):
        import torch
        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.sink)


def launches_per_step(w):
    """This library's kernels per step: the quantize (or rotate + quantize) launch, then
    the attention call: the split-KV decode kernel (its last CTA per head combines the
    partials), or for prefill the V' pre-pass and the attention kernel (mixed branches: one
    bf16 dequantize launch per quantized Q / K first)."""
    if w.name == "int8_decode":
        return 1 + 1
    if w.branch_modes is not None:
        return 1 + sum(m != "float" for m in w.branch_modes[:2]) + 2
    return 1 + 2


def attention_kernels(w):
    """(label, source file) of the attention call's kernels for this workload."""
    if w.name == "int8_decode":
        return "decode_kernel with the LSE combine fused (one fa_attention_quant call)", "decode.cu"
    if w.branch_modes is not None:
        return "deq_bf16_kernel x2 + vprep_kernel + attn_pair_kernel<bf16> (one fa_attention_quant call)", "attn2.cu"
    if w.mode in ("mxfp4", "mxfp8"):
        return "vprep_kernel + attn_pair_kernel<MX, 112-key tiles> (one fa_attention_quant call)", "attn2.cu"
    return "vprep_kernel + attn_pair_kernel (one fa_attention_quant call)", "attn2.cu"


def max_over_ranks(vals, world, device):
    """Each rank's timed sums -> their maxima over ranks (the slowest rank sets the job's
    time).  One all-reduce on the process group; identity for one rank."""
    if world == 1:
        return [float(x) for x in vals]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x) for x in vals], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_value(work_per_rank, ms_per_step, world, unit):
    """Whole-job throughput: every rank processes work_per_rank units per step (weak scaling),
    the step takes ms_per_step on the slowest rank."""
    return world * work_per_rank / (ms_per_step * 1e-3) / (1e9 if unit == "GB/s" else 1e12)


def gpu_run(args, w, rank, world, device):
    import torch
    import quantized_attention_amax_b200 as faq
    import workloads as wl

    torch.cuda.set_device(device)
    step, attn, quant, st = make_step(faq, wl, w, device, seed_offset=rank)
    flush = L2Flush(device)
    stream = torch.cuda.current_stream()
    for _ in range(max(args.warmup, 3)):
        step()
    faq.check_device_status()
    torch.cuda.synchronize()
    # CUDA graphs: one for the quantize launch, one for attention
    gq, ga = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(stream)
    with torch.cuda.stream(s):
        quant()
        attn()
    stream.wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(gq):
        quant()
    with torch.cuda.graph(ga):
        attn()
    for _ in range(max(args.warmup, 3)):
        flush()
        gq.replay()
        ga.replay()
    torch.cuda.synchronize()
    faq.check_device_status()

    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(device).uuid)
        uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        uuid = None
    clocks = ClockSampler(uuid)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.25)
    t0 = time.perf_counter()
    for i in range(K):
        flush()
        ev[i][0].record(stream)
        gq.replay()
        ev[i][1].record(stream)
        ga.replay()
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    faq.check_device_status()
    q_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(K)]
    a_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(K)]
    total_ms, a_sum, q_sum = max_over_ranks([sum(q_ms) + sum(a_ms), sum(a_ms), sum(q_ms)], world, device)
    res = {"total_ms": total_ms, "attn_ms": a_sum / K, "quant_ms": q_sum / K, "wall_s": wall, "clocks": clk,
           "st": st, "step": step}
    return res


def e2e_run(args, w, device, steps):
    """Same metric through the public API with pinned host buffers: every step copies its
    bf16 inputs host -> device, runs quantize + attention, and reads its output back to the
    host.  Steps are pipelined the way a serving loop runs them: the copies run on their own
    streams (one per direction) into double buffers, so step i+1's inputs and step i-1's
    output cross PCIe while step i computes."""
    import torch
    import quantized_attention_amax_b200 as faq
    import workloads as wl

    inp = wl.make_inputs(w, device="cpu", calib=(w.mode in STATIC_MODES))
    host = {n: inp[n].pin_memory() for n in ("q", "k", "v")}
    dev = [{n: torch.empty_like(host[n], device=device) for n in host} for _ in range(2)]
    R = inp["R"].to(device) if inp.get("R") is not None else None
    signs = wl.rotation_signs(w.D, w.seed) if w.rotate else None
    amax = None
    if w.mode in STATIC_MODES:
        amax = [faq.calibrate_per_head(inp[n + "_cal"].to(device), w.layout) for n in "qkv"]
    out_h = [torch.empty_like(host["q"]).pin_memory() for _ in range(2)]
    out_d = [torch.empty_like(host["q"], device=device) for _ in range(2)]
    decode = w.name == "int8_decode"
    cache = None
    if decode:
        for n in ("k", "v"):
            dev[0][n].copy_(host[n])
        cache = faq.quantize(None, dev[0]["k"], dev[0]["v"], w.mode, w.layout, amax=[None, amax[1], amax[2]])
    names = ("q",) if decode else ("q", "k", "v")
    s_in, s_cmp, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()
    in_ready, cmp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for e in cmp_done + out_done:
        e.record(torch.cuda.current_stream(device))
    ws = None

    def one(i):
        nonlocal ws
        b = i & 1
        d = dev[b]
        with torch.cuda.stream(s_in):
            s_in.wait_event(cmp_done[b])  # step i-2 has finished reading this buffer
            for n in names:
                d[n].copy_(host[n], non_blocking=True)
            in_ready[b].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(in_ready[b])
            s_cmp.wait_event(out_done[b])  # step i-2's output has left this buffer
            if decode:
                Q = faq.quantize(d["q"], None, None, w.mode, w.layout, amax=[amax[0], None, None])[0]
                K, V = cache[1], cache[2]
            elif w.rotate and ROTATION == "hadamard":
                Q, K, V = faq.rotate_quantize_hadamard(d["q"], d["k"], d["v"], signs, signs, w.layout, w.q_block,
                                                       w.kv_block)
            elif w.rotate:
                Q, K, V = faq.rotate_quantize(d["q"], d["k"], d["v"], R, R, w.layout, w.q_block, w.kv_block)
            elif amax is not None:
                Q, K, V = faq.quantize(d["q"], d["k"], d["v"], w.mode, w.layout, amax=amax)
            else:
                Q, K, V = faq.quantize(d["q"], d["k"], d["v"], w.mode, w.layout, q_block=w.q_block,
                                       kv_block=w.kv_block)
            if ws is None:
                nb = faq.attention_workspace_size(Q, K)
                ws = torch.empty(max(nb, 16), dtype=torch.uint8, device=device)
            faq.attention(Q, K, V, causal=w.causal, workspace=ws, out=out_d[b])
            cmp_done[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(cmp_done[b])
            out_h[b].copy_(out_d[b], non_blocking=True)
            out_done[b].record(s_out)

    for i in range(2):
        one(i)
    torch.cuda.synchronize(device)
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for i in range(steps):
        one(i)
    s_in.wait_stream(s_out)
    s_in.wait_stream(s_cmp)
    z.record(s_in)
    torch.cuda.synchronize(device)
    ms = a.elapsed_time(z) / steps
    h2d = sum(host[n].numel() * 2 for n in names)
    d2h = out_h[0].numel() * 2
    return ms, h2d, d2h


# --------------------------------------------------------- oracle / CPU ---

def sample_rows(w, n=256, seed=0):
    """Query rows of the oracle's sample: the first and last rows, the tile boundaries
    127/128/255/256, and seeded random rows up to n (all rows when Sq <= n)."""
    import numpy as np
    if w.Sq <= n:
        return list(range(w.Sq))
    fixed = [r for r in (0, 127, 128, 255, 256, w.Sq - 1) if r < w.Sq]
    rest = [r for r in np.random.default_rng(seed).permutation(w.Sq).tolist() if r not in fixed]
    return sorted(fixed + rest[:n - len(fixed)])


def oracle_sample(w, reps_seconds=None):
    """The oracle on a bounded sample of the workload: quantize one GQA group
    (batch 0, kv head 0 and its query heads: the whole Q/K/V of the group)
    and attention for 256 sampled query rows of each of its heads (every row
    when the sequence is shorter).  Rows are independent, so the sample's
    time extrapolates to the whole workload by its share of the unmasked
    (query, key) pairs.  Returns (run_once, FLOPs or bytes per sample,
    description, full-workload work / sample work)."""
    import numpy as np
    import oracle as orc
    import workloads as wl

    G = w.Hq // w.Hkv
    rows = sample_rows(w)
    sub = w.scaled(B=1, Hq=G, Hkv=1)
    inp = wl.make_inputs(sub, calib=(w.mode in STATIC_MODES))
    qb = wl.bf16_bits(inp["q"])
    kb = wl.bf16_bits(inp["k"])
    vb = wl.bf16_bits(inp["v"])
    L = w.layout
    amax = None
    if w.mode in STATIC_MODES:
        amax = {n: orc.calibrate_per_head(wl.bf16_bits(inp[n + "_cal"]), L) for n in "qkv"}
    Rb = wl.bf16_bits(inp["R"]) if inp.get("R") is not None else None

    def run_once():
        t0 = time.perf_counter()
        if w.mode == "int8_per_head":
            cq, sq = orc.quantize_int8_per_head(qb, amax["q"], L)
            ck, sk = orc.quantize_int8_per_head(kb, amax["k"], L)
            cv, sv = orc.quantize_int8_per_head(vb, amax["v"], L)
            blks = (0, 0, 0)
        elif w.mode == "fp8_per_head":
            (cq, sq), (ck, sk), (cv, sv) = (orc.quantize_fp8_per_head(x, amax[n], L) for x, n in zip((qb, kb, vb), "qkv"))
            blks = (0, 0, 0)
        elif w.mode == "int8_per_token":
            (cq, sq), (ck, sk), (cv, sv) = (orc.quantize_int8_per_token(x, L) for x in (qb, kb, vb))
            blks = (0, 0, 0)
        elif w.mode == "fp8_per_token":
            (cq, sq), (ck, sk), (cv, sv) = (orc.quantize_fp8_per_token(x, L) for x in (qb, kb, vb))
            blks = (0, 0, 0)
        elif w.mode == "mxfp4":
            (cq, sq), (ck, sk), (cv, sv) = (orc.quantize_mxfp4(x, L) for x in (qb, kb, vb))
            blks = (0, 0, 0)
        elif w.mode == "mxfp8":
            (cq, sq), (ck, sk), (cv, sv) = (orc.quantize_mxfp8(x, L) for x in (qb, kb, vb))
            blks = (0, 0, 0)
        else:
            qr = orc.rotate(qb, Rb, L) if Rb is not None else qb
            kr = orc.rotate(kb, Rb, L) if Rb is not None else kb
            cq, sq = orc.quantize_fp8_block(qr, w.q_block, L)
            ck, sk = orc.quantize_fp8_block(kr, w.kv_block, L)
            cv, sv = orc.quantize_fp8_block(vb, w.kv_block, L)
            blks = (w.q_block, w.kv_block, w.kv_block)
        Q = orc.QT(w.mode, cq, sq, 1, G, w.Sq, w.D, L, blks[0])
        K = orc.QT(w.mode, ck, sk, 1, 1, w.Sk, w.D, L, blks[1])
        V = orc.QT(w.mode, cv, sv, 1, 1, w.Sk, w.D, L, blks[2])
        orc.attention(Q, K, V, w.causal, 0.0, rows)
        return time.perf_counter() - t0

    diag = w.Sk - w.Sq
    pairs = sum((max(0, min(w.Sk, i + diag + 1)) if w.causal else w.Sk) for i in rows) * G
    work = 4.0 * w.D * pairs
    full = attn_flops(w)
    if w.name == "int8_decode":
        work = 2.0 * w.Sk * w.D  # KV bytes of one kv head
        full = decode_bytes(w)
    desc = (f"one GQA group (batch 0, kv head 0, its {G} query heads): quantize its Q/K/V "
            f"({'rotate + ' if Rb is not None else ''}{w.mode}) and attention for {len(rows)} query rows "
            f"of each head (rows 0, 127, 128, 255, 256, {w.Sq - 1} and seeded random rows); the rate "
            f"extrapolates to the whole workload by its unmasked (query, key) pairs")
    return run_once, work, desc, full / work


def cpu_baseline(w, seconds=8.0):
    import oracle as orc
    run_once, work, desc, scale = oracle_sample(w)
    run_once()  # builds the oracle, warms caches
    ts = []
    t_end = time.perf_counter() + seconds
    while time.perf_counter() < t_end or len(ts) < 2:
        ts.append(run_once())
    per = statistics.median(ts)
    unit = "GB/s" if w.name == "int8_decode" else "TFLOP/s"
    val = work / per / (1e9 if unit == "GB/s" else 1e12)
    return {"value": val, "unit": unit, "cores": orc.num_threads(), "kind": "oracle", "sample": desc,
            "seconds_per_sample": per, "samples": len(ts),
            "extrapolated_step_s": per * scale, "extrapolated": True}


def reference_arm(args, w):
    import oracle as orc
    run_once, work, desc, scale = oracle_sample(w)
    for _ in range(max(args.warmup, 0)):
        run_once()
    ts = [run_once() for _ in range(args.steps)]
    total = sum(ts)
    unit = "GB/s" if w.name == "int8_decode" else "TFLOP/s"
    val = work * args.steps / total / (1e9 if unit == "GB/s" else 1e12)
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
            "data": DATA[w.name], "config": {"workload": f"{w.name}: {DESCR[w.name]}", "sample": desc},
            "cpu_baseline": {"value": val, "unit": unit, "cores": orc.num_threads(), "kind": "oracle",
                             "sample": desc, "extrapolated_step_s": total / args.steps * scale,
                             "extrapolated": True},
            "e2e": {"value": val, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ main ---

def decode_append_run(w, device, steps):
    """fa_decode_append on the decode workload's cache: each step quantizes the query, appends the
    last token's K / V into the cache and attends over all Sk tokens (one call, two launches)."""
    import torch
    import quantized_attention_amax_b200 as faq
    import workloads as wl
    inp = wl.make_inputs(w, device=device, calib=True)
    am = [faq.calibrate_per_head(inp[n + "_cal"], w.layout) for n in "qkv"]
    _, Kc, Vc = faq.quantize(None, inp["k"], inp["v"], w.mode, w.layout, amax=[None, am[1], am[2]])
    pos = w.Sk - 1
    k_new = inp["k"][:, :, pos:pos + 1].contiguous()
    v_new = inp["v"][:, :, pos:pos + 1].contiguous()
    out = faq.decode_append(inp["q"], k_new, v_new, am, Kc, Vc, pos)
    ws = torch.empty(1 << 24, dtype=torch.uint8, device=device)
    fn = lambda: faq.decode_append(inp["q"], k_new, v_new, am, Kc, Vc, pos, out=out, workspace=ws)
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    with torch.cuda.graph(g):
        fn()
    flush = L2Flush(device)
    stream = torch.cuda.current_stream()
    ms = []
    for i in range(steps + 3):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        b.synchronize()
        if i >= 3:
            ms.append(a.elapsed_time(b))
    faq.check_device_status()
    return sum(ms) / len(ms)


def supplemental(args, device):
    """Every other workload, briefly (graph replays, L2 flushed): kernel-level
    numbers against their rooflines.  Context for the headline line."""
    import workloads as wl
    out = {}
    pk = peaks()
    for name in ("int8_tiny", "rot_fp8_block", "mxfp4", "int8_decode", "int8_prefill", "fp8_head_prefill",
                 "int8_token_prefill", "mxfp8", "mixed_prefill"):
        w = wl.WORKLOADS[name]
        a = argparse.Namespace(steps=10 if name != "rot_fp8_block" else 4, warmup=3)
        r = gpu_run(a, w, 0, 1, device)
        d = {"ms_per_step": r["total_ms"] / a.steps, "attn_ms": r["attn_ms"], "quant_ms": r["quant_ms"]}
        qb = quant_bytes(w)
        d["quantize"] = {"GB/s": qb / (r["quant_ms"] * 1e-3) / 1e9,
                         "frac_of_hbm": qb / (r["quant_ms"] * 1e-3) / 1e9 / pk["hbm_gbs"], "bytes": qb}
        if name == "int8_decode":
            db = decode_bytes(w)
            d["value"] = db / (r["attn_ms"] * 1e-3) / 1e9
            d["unit"] = "GB/s (KV codes)"
            d["attention"] = {"GB/s": d["value"], "frac_of_hbm": d["value"] / pk["hbm_gbs"], "bytes": db}
        else:
            fl = attn_flops(w)
            tp = tensor_peak(w, pk)
            d["value"] = fl / (r["total_ms"] / a.steps * 1e-3) / 1e12
            d["unit"] = "TFLOP/s (step)"
            d["attention"] = {"TFLOP/s": fl / (r["attn_ms"] * 1e-3) / 1e12,
                              "frac_of_peak": fl / (r["attn_ms"] * 1e-3) / 1e12 / tp, "peak": tp, "flops": fl}
        out[name] = d
        del r
    w = wl.WORKLOADS["int8_decode"]
    ams = decode_append_run(w, device, 10)
    db = decode_bytes(w)
    out["int8_decode_append"] = {
        "ms_per_step": ams, "unit": "GB/s (KV codes)", "value": db / (ams * 1e-3) / 1e9,
        "attention": {"GB/s": db / (ams * 1e-3) / 1e9, "frac_of_hbm": db / (ams * 1e-3) / 1e9 / pk["hbm_gbs"],
                      "bytes": db},
        "note": "fa_decode_append: query quantize + K/V append at position Sk-1 + split-KV decode + combine, "
                "two launches per step"}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=600)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="faq", choices=["faq", "reference"])
    ap.add_argument("--workload", default="fp8_prefill")
    ap.add_argument("--no-supplemental", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--rotation", default="matrix", choices=["matrix", "hadamard"],
                    help="rotating workloads: R from memory, or the same R given by its signs")
    args = ap.parse_args()
    global ROTATION
    ROTATION = args.rotation

    import workloads as wl
    w = wl.WORKLOADS[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            reference_arm(args, w)
        return

    import torch
    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}))
        sys.exit(1)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    from quantized_attention_amax_b200 import build
    if rank == 0 or world == 1:
        build.build()
    if world > 1:
        dist.barrier()

    r = gpu_run(args, w, rank, world, device)
    K = args.steps
    pk = peaks()
    ms_per_step = r["total_ms"] / K
    if w.name == "int8_decode":
        unit = "GB/s"
        work = decode_bytes(w)
    else:
        unit = "TFLOP/s"
        work = attn_flops(w)
    value = job_value(work, ms_per_step, world, unit)

    # dominant kernel: attention
    if unit == "GB/s":
        ach = work / (r["attn_ms"] * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": ach / pk["hbm_gbs"],
                "traffic": None, "kernel": attention_kernels(w)[0],
                "peak_source": f"{pk['src']} HBM copy bandwidth"}
    else:
        tp = tensor_peak(w, pk)
        ach = work / (r["attn_ms"] * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": tp, "unit": "TFLOP/s", "frac": ach / tp,
                "traffic": None, "kernel": attention_kernels(w)[0],
                "peak_source": (f"{pk['src']} bf16 burst (mixed branches: QK^T on bf16)" if w.branch_modes is not None
                                else f"{pk['src']} bf16 burst x {4 if w.mode == 'mxfp4' else 2} (dense "
                                     f"{'FP4' if w.mode == 'mxfp4' else 'FP8/INT8'} : bf16 nominal ratio)")}
    prof = os.path.join(ROOT, "profiles", f"traffic_{w.name}.json")
    if os.path.exists(prof):
        # DRAM bytes per launch from one ncu capture, valid only while the
        # kernel source is the one that was captured.
        try:
            import hashlib
            tr = json.load(open(prof))
            src = os.path.join(ROOT, "quantized_attention_amax_b200", "csrc",
                               tr.get("kernel_source", attention_kernels(w)[1]))
            sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
            if sha == tr.get("attn_cu_sha256_16"):
                roof["traffic"] = tr.get("dram_bytes_per_launch")
                roof["traffic_source"] = tr.get("source")
        except Exception:
            pass

    line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": DTYPE[w.name], "data": DATA[w.name],
            "config": {"workload": f"{w.name}: {DESCR[w.name]}",
                       "l2": "flushed between steps (256 MiB device write, then a 256 MiB read so no dirty "
                             "line of the flush is left; outside the timed events)",
                       "timing": "CUDA-graph replay per launch, CUDA events on the launch stream",
                       "parallelism": f"replicas x{world} (independent workloads per rank)",
                       **({"rotation": "R from memory (fa_rotate_quantize)" if ROTATION == "matrix" else
                           "R = bf16(H diag(signs) / sqrt(D)) from its signs (fa_rotate_quantize_hadamard)"}
                          if w.rotate else {})},
            "kernels_ms": {"quantize": r["quant_ms"], "attention": r["attn_ms"]},
            "quantize_roofline": {"bound": "hbm", "achieved": quant_bytes(w) / (r["quant_ms"] * 1e-3) / 1e9,
                                  "peak": pk["hbm_gbs"], "unit": "GB/s",
                                  "frac": quant_bytes(w) / (r["quant_ms"] * 1e-3) / 1e9 / pk["hbm_gbs"]},
            "roofline": roof, "gpu_launches": K * launches_per_step(w), "clocks": r["clocks"]}
    del r["st"]
    if rank == 0:
        if not args.no_e2e:
            ems, h2d, d2h = e2e_run(args, w, device, steps=20)
            e2e_val = work / (ems * 1e-3) / (1e9 if unit == "GB/s" else 1e12)
            line["e2e"] = {"value": e2e_val, "unit": unit, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                           "ms_per_step": ems, "path": "pinned host -> public Python API (C-ABI) -> pinned host; copies on their own streams, overlapped with the neighbouring steps' compute"}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
        if world == 1 and not args.no_supplemental:
            line["supplemental"] = supplemental(args, device)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
