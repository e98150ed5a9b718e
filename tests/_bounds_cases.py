"""Small ragged cases through every entry point, for the bounds-checked build test: run as
    FAQ_LIB=bounds python tests/_bounds_cases.py OUT.npz
(or without FAQ_LIB for the ordinary build); saves every output and exits non-zero if the device
status reports anything.  Inputs are seeded; shapes are off the tile sizes on purpose."""
import os
import sys

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
import quantized_attention_amax_b200 as faq  # noqa: E402
import workloads as wl  # noqa: E402


def main(path):
    out = {}
    dev = "cuda"

    def keep(name, t):
        out[name] = t.detach().float().cpu().numpy() if t.dtype != torch.uint8 and t.dtype != torch.int8 \
            else t.detach().cpu().numpy()

    for mode in ("fp8_per_token", "int8_per_token", "mxfp4", "mxfp8", "fp8_block"):
        for layout, D, S in (("BNSD", 128, 300), ("BSND", 64, 257)):
            if mode.startswith("mx") and D != 128:
                continue
            shp = (1, 3, S, D) if layout == "BNSD" else (1, S, 3, D)
            kshp = (1, 1, S, D) if layout == "BNSD" else (1, S, 1, D)
            q = wl.normal(shp, 1).to(dev)
            k = wl.normal_k_outliers(kshp, layout, 2).to(dev)
            v = wl.normal(kshp, 3).to(dev)
            Q, K, V = faq.quantize(q, k, v, mode, layout, q_block=64, kv_block=128)
            o = faq.attention(Q, K, V, causal=True)
            tag = f"{mode}_{layout}_{D}"
            keep(tag + "_qc", Q.codes)
            keep(tag + "_qs", Q.scales)
            keep(tag + "_out", o)
    for mode in ("int8_per_head", "fp8_per_head"):
        q = wl.normal((2, 4, 130, 128), 4).to(dev)
        k = wl.normal((2, 2, 130, 128), 5).to(dev)
        v = wl.normal((2, 2, 130, 128), 6).to(dev)
        am = [faq.calibrate_per_head(x) for x in (q, k, v)]
        Q, K, V = faq.quantize(q, k, v, mode, amax=am)
        o = faq.attention(Q, K, V, causal=False)
        keep(mode + "_kc", K.codes)
        keep(mode + "_out", o)
    # rotation (stored R and Hadamard signs), and the FWHT kernel's block sizes
    q = wl.normal((1, 300, 2, 128), 7).to(dev)
    k = wl.normal((1, 300, 2, 128), 8).to(dev)
    v = wl.normal((1, 300, 2, 128), 9).to(dev)
    R = wl.rotation(128, 3).to(dev)
    Q, K, V = faq.rotate_quantize(q, k, v, R, R, "BSND", 128, 256)
    keep("rot_q", Q.codes)
    sg = wl.rotation_signs(128, 3)
    for qb, kb in ((128, 256), (100, 300)):
        Q, K, V = faq.rotate_quantize_hadamard(q, k, v, sg, sg, "BSND", qb, kb)
        keep(f"had_{qb}_k", K.codes)
        keep(f"had_{qb}_ks", K.scales)
    # INT8 decode
    q = wl.normal((3, 8, 1, 128), 10).to(dev)
    k = wl.normal((3, 2, 1000, 128), 11).to(dev)
    v = wl.normal((3, 2, 1000, 128), 12).to(dev)
    am = [faq.calibrate_per_head(x) for x in (q, k, v)]
    Q, K, V = faq.quantize(q, k, v, "int8_per_head", amax=am)
    o = faq.attention(Q, K, V, causal=False)
    keep("decode_out", o)
    faq.check_device_status()
    np.savez(path, **out)


if __name__ == "__main__":
    main(sys.argv[1])
