"""The C-ABI library loads, exports every symbol include/faq.h declares, and
rejects bad arguments on the host before any CUDA call (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def N():
    from quantized_attention_amax_b200 import build
    build.build()
    from quantized_attention_amax_b200 import _native
    _native.lib()
    return _native


def declared_symbols():
    hdr = open(os.path.join(ROOT, "include", "faq.h")).read()
    return sorted(set(re.findall(r"FAQ_API\s+[\w\s\*]*?\b(fa_\w+)\s*\(", hdr)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("fa_calibrate_per_head", "fa_quantize", "fa_rotate_quantize", "fa_attention_quant"):
        assert name in syms


def test_library_exports_every_declared_symbol(N):
    out = subprocess.run(["nm", "-D", "--defined-only", N.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (fa_\w+)", out))
    assert set(declared_symbols()) <= exported
    assert set(N.EXPORTS) == set(declared_symbols())
    L = N.lib()
    for name in declared_symbols():
        assert getattr(L, name) is not None


def test_status_strings(N):
    L = N.lib()
    for code in range(9):
        assert L.fa_status_str(code)
    assert L.fa_status_str(8) != L.fa_status_str(99)  # FA_ERR_BOUNDS has its own text
    assert b"x" in L.fa_version() or L.fa_version()


def test_bounds_checked_build_exports_the_same_boundary():
    """The FA_DEBUG_BOUNDS build (index checks that set the status word instead of faulting)
    compiles from the same sources and exports the same symbols."""
    from quantized_attention_amax_b200 import build
    path = build.build(bounds=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (fa_\w+)", out))
    assert set(declared_symbols()) <= exported


def test_resolve_config_rules():
    import quantized_attention_amax_b200 as faq
    # neither given: the default int8 / per_head
    assert faq.resolve_config() == ("int8_per_head",) * 3
    assert faq.resolve_config("fp8_per_token") == ("fp8_per_token",) * 3
    assert faq.resolve_config(details=["fp8_per_head", "int8_per_token", None]) == ("fp8_per_head", "int8_per_token",
                                                                                     "float")
    # a branch details leaves unset stays float
    assert faq.resolve_config(details=["mxfp4", None, None]) == ("mxfp4", "float", "float")
    with pytest.raises(faq.FaqError) as e:
        faq.resolve_config("int8_per_head", ["int8_per_head", None, None])
    assert e.value.status == 4


def _t(N, B=1, H=2, S=8, D=64, layout=0, ptr=0x10000):
    return N.FaTensor(ptr, B, H, S, D, layout)


def _q(N, mode, B=1, H=2, S=8, D=64, layout=0, blk=0, codes=0x20000, scales=0x30000):
    return N.FaQTensor(codes, scales, mode, B, H, S, D, layout, blk)


def test_quantize_validation_before_launch(N):
    L = N.lib()
    t = _t(N)
    o = _q(N, 2)
    by = ctypes.byref
    assert L.fa_quantize(by(t), None, None, 0, None, None, None, by(o), None, None, None) == 1   # float mode
    t96 = _t(N, D=96)
    o96 = _q(N, 2, D=96)
    assert L.fa_quantize(by(t96), None, None, 2, None, None, None, by(o96), None, None, None) == 2  # D
    oi = _q(N, 1)
    assert L.fa_quantize(by(t), None, None, 1, None, None, None, by(oi), None, None, None) == 3  # no calibration
    oh = _q(N, 5)  # FA PerHead FP8 is static too
    assert L.fa_quantize(by(t), None, None, 5, None, None, None, by(oh), None, None, None) == 3
    assert L.fa_quantize(by(t), None, None, 6, None, None, None, by(oh), None, None, None) == 1  # mode mismatch
    assert L.fa_quantize(by(t), None, None, 8, None, None, None, by(oh), None, None, None) == 2  # unknown mode
    bad = _q(N, 2, S=9)
    assert L.fa_quantize(by(t), None, None, 2, None, None, None, by(bad), None, None, None) == 1  # shape mismatch
    mis = _t(N, ptr=0x10008)
    assert L.fa_quantize(by(mis), None, None, 2, None, None, None, by(o), None, None, None) == 1  # alignment
    ob = _q(N, 4, blk=0)
    assert L.fa_quantize(by(t), None, None, 4, None, None, None, by(ob), None, None, None) == 1  # block size
    assert L.fa_quantize(None, None, None, 2, None, None, None, None, None, None, None) == 1     # nothing to do
    assert L.fa_calibrate_per_head(by(t96), ctypes.c_void_p(0x40000), None) == 2
    assert L.fa_calibrate_per_head(by(t), None, None) == 1


def test_rotate_validation_before_launch(N):
    L = N.lib()
    by = ctypes.byref
    t = _t(N)
    oq, ok, ov = _q(N, 4, blk=128), _q(N, 4, blk=256), _q(N, 4, blk=256)
    # missing rotation matrix
    assert L.fa_rotate_quantize(by(t), by(t), by(t), None, None, 128, 256, by(oq), by(ok), by(ov),
                                None, None, None) == 1
    # block size disagreeing with the output descriptor
    assert L.fa_rotate_quantize(by(t), by(t), by(t), 0x50000, 0x50000, 64, 256, by(oq), by(ok), by(ov),
                                None, None, None) == 1
    # wrong output mode
    om = _q(N, 2)
    assert L.fa_rotate_quantize(by(t), by(t), by(t), 0x50000, 0x50000, 128, 256, by(om), by(ok), by(ov),
                                None, None, None) == 1


def test_attention_validation_before_launch(N):
    L = N.lib()
    by = ctypes.byref
    q = _q(N, 2, H=4)
    k = _q(N, 2, H=2)
    v = _q(N, 2, H=2)
    km = _q(N, 1, H=2)
    # mixed branches run (the bf16 path): without a workspace they stop at the workspace check
    assert L.fa_attention_quant(by(q), by(km), by(v), 0, 0.0, 0x60000, None, 0, None, 0, None) == 7  # mixed
    k3 = _q(N, 2, H=3)
    assert L.fa_attention_quant(by(q), by(k3), by(k3), 0, 0.0, 0x60000, None, 0, None, 0, None) == 1  # GQA
    kd = _q(N, 2, H=2, D=128)
    assert L.fa_attention_quant(by(q), by(kd), by(kd), 0, 0.0, 0x60000, None, 0, None, 0, None) == 1  # D
    assert L.fa_attention_quant(by(q), by(k), by(v), 0, 0.0, None, None, 0, None, 0, None) == 1      # out
    qf = _q(N, 0, H=4)
    assert L.fa_attention_quant(by(qf), by(k), by(v), 0, 0.0, 0x60000, None, 0, None, 0, None) == 7  # float
    # decode without workspace
    qd = _q(N, 1, B=2, H=4, S=1, D=128)
    kd = _q(N, 1, B=2, H=2, S=1000, D=128)
    need = L.fa_attention_workspace_size(by(qd), by(kd), 0)
    assert need > 0
    assert L.fa_attention_quant(by(qd), by(kd), by(kd), 0, 0.0, 0x60000, None, 0, None, 0, None) == 7
    assert L.fa_attention_quant(by(qd), by(kd), by(kd), 0, 0.0, 0x60000, None, 0, 0x70000, need - 16,
                                None) == 7
    assert L.fa_attention_quant(by(qd), by(kd), by(kd), 0, 0.0, 0x60000, None, -1, None, 0, None) == 1
    # prefill: fp16 V', a 16-byte factor record and 512 bytes of K scales per 128-key tile,
    # each part 256-byte aligned
    qp = _q(N, 1, B=2, H=4, S=100, D=128)
    need_p = L.fa_attention_workspace_size(by(qp), by(kd), 0)
    ntiles = (1000 + 127) // 128
    parts = (2 * 2 * 1000 * 128 * 2, 2 * 2 * ntiles * 16, 2 * 2 * ntiles * 128 * 4)
    assert need_p == sum(((x + 255) // 256) * 256 for x in parts)
    assert L.fa_attention_quant(by(qp), by(kd), by(kd), 0, 0.0, 0x60000, None, 0, None, 0, None) == 7
    assert L.fa_attention_quant(by(qp), by(kd), by(kd), 0, 0.0, 0x60000, None, 0, 0x70000, need_p - 256,
                                None) == 7
    assert L.fa_attention_quant(by(qp), by(kd), by(kd), 0, 0.0, 0x60000, None, 0, 0x70010, need_p,
                                None) == 7  # workspace not 256-byte aligned
    # the FA PerHead FP8 / PerToken INT8 modes use the same prefill workspace
    for m in (5, 6):
        assert L.fa_attention_workspace_size(by(_q(N, m, B=2, H=4, S=100, D=128)), by(_q(N, m, B=2, H=2, S=1000, D=128)),
                                             0) == need_p
    # MXFP4 / MXFP8 prefill: the same parts over 112-key tiles (their K scales are the tile's
    # scale-factor atom); head_dim 128 only
    ntiles_mx = (1000 + 111) // 112
    parts_mx = (2 * 2 * 1000 * 128 * 2, 2 * 2 * ntiles_mx * 16, 2 * 2 * ntiles_mx * 128 * 4)
    need_mx = sum(((x + 255) // 256) * 256 for x in parts_mx)
    assert need_mx > need_p
    assert L.fa_attention_workspace_size(by(_q(N, 7, B=2, H=4, S=100, D=128)), by(_q(N, 7, B=2, H=2, S=1000, D=128)),
                                         0) == need_mx
    qm = _q(N, 3, B=2, H=4, S=100, D=128)
    km = _q(N, 3, B=2, H=2, S=1000, D=128)
    assert L.fa_attention_workspace_size(by(qm), by(km), 0) == need_mx
    assert L.fa_attention_quant(by(qm), by(km), by(km), 0, 0.0, 0x60000, None, 0, None, 0, None) == 7
    qm64, km64 = _q(N, 3, B=2, H=4, S=100, D=64), _q(N, 3, B=2, H=2, S=1000, D=64)
    assert L.fa_attention_workspace_size(by(qm64), by(km64), 0) == 0
    assert L.fa_attention_quant(by(qm64), by(km64), by(km64), 0, 0.0, 0x60000, None, 0, None, 0, None) == 2
    # scales that are not 4-byte aligned are rejected on the host, for every operand and mode
    for m in (1, 2, 3, 4, 5, 6, 7):
        blk = 256 if m == 4 else 0
        qa = _q(N, m, B=2, H=4, S=100, D=128, blk=blk)
        ka = _q(N, m, B=2, H=2, S=1000, D=128, blk=blk)
        kmis = _q(N, m, B=2, H=2, S=1000, D=128, blk=blk, scales=0x30002)
        qmis = _q(N, m, B=2, H=4, S=100, D=128, blk=blk, scales=0x30001)
        assert L.fa_attention_quant(by(qa), by(kmis), by(ka), 0, 0.0, 0x60000, None, 0, 0x70000, 1 << 40, None) == 1
        assert L.fa_attention_quant(by(qa), by(ka), by(kmis), 0, 0.0, 0x60000, None, 0, 0x70000, 1 << 40, None) == 1
        assert L.fa_attention_quant(by(qmis), by(ka), by(ka), 0, 0.0, 0x60000, None, 0, 0x70000, 1 << 40, None) == 1


def test_noalloc_validation_before_launch(N):
    """The allocation-free decode checks its arguments like fa_attention_quant: misaligned scales
    are rejected before any launch, and a batch of zero is a successful no-op."""
    L = N.lib()
    by = ctypes.byref
    qd = _q(N, 1, B=2, H=4, S=1, D=128)
    kd = _q(N, 1, B=2, H=2, S=1000, D=128)
    for bad in (_q(N, 1, B=2, H=2, S=1000, D=128, scales=0x30002),):
        assert L.fa_attention_decode_noalloc(by(qd), by(bad), by(kd), 0.0, 0x60000, None, 0, None) == 1
        assert L.fa_attention_decode_noalloc(by(qd), by(kd), by(bad), 0.0, 0x60000, None, 0, None) == 1
    qmis = _q(N, 1, B=2, H=4, S=1, D=128, scales=0x30001)
    assert L.fa_attention_decode_noalloc(by(qmis), by(kd), by(kd), 0.0, 0x60000, None, 0, None) == 1
    assert L.fa_attention_decode_noalloc(by(qd), by(kd), by(kd), 0.0, 0x60008, None, 0, None) == 1  # out
    q0, k0 = _q(N, 1, B=0, H=4, S=1, D=128), _q(N, 1, B=0, H=2, S=1000, D=128)
    assert L.fa_attention_decode_noalloc(by(q0), by(k0), by(k0), 0.0, None, None, 0, None) == 0
    assert L.fa_attention_decode_noalloc(by(qd), by(kd), by(kd), 0.0, 0x60000, None, -1, None) == 1
    # partials beyond the fixed buffer: B * Hq * splits * (D + 2) * 4 bytes > 16 MiB
    assert L.fa_attention_decode_noalloc(by(qd), by(kd), by(kd), 0.0, 0x60000, None, 5000, None) == 7


def test_mixed_branch_validation_and_workspace(N):
    """Per-branch modes (fa3_quant details): a float branch is the bf16 tensor itself; mixed
    calls need V' parts plus bf16 copies of the Q / K branches that are quantized."""
    L = N.lib()
    by = ctypes.byref
    B, Hq, Hkv, Sq, Sk, D = 2, 4, 2, 100, 1000, 128
    ntiles = (Sk + 127) // 128
    r256 = lambda x: ((x + 255) // 256) * 256
    base = sum(r256(x) for x in (B * Hkv * Sk * D * 2, B * Hkv * ntiles * 16, B * Hkv * ntiles * 128 * 4))
    qcopy, kcopy = r256(B * Hq * Sq * D * 2), r256(B * Hkv * Sk * D * 2)
    q8, k8 = _q(N, 2, B=B, H=Hq, S=Sq, D=D), _q(N, 2, B=B, H=Hkv, S=Sk, D=D)
    qf, kf, vf = _q(N, 0, B=B, H=Hq, S=Sq, D=D), _q(N, 0, B=B, H=Hkv, S=Sk, D=D), _q(N, 0, B=B, H=Hkv, S=Sk, D=D)
    ki = _q(N, 1, B=B, H=Hkv, S=Sk, D=D)
    # all three float: plain bf16 attention, nothing to dequantize
    assert L.fa_attention_workspace_size_qkv(by(qf), by(kf), by(vf), 0) == base
    # Q quantized, K float: Q's bf16 copy only
    assert L.fa_attention_workspace_size_qkv(by(q8), by(kf), by(vf), 0) == base + qcopy
    # Q and K in different modes: both copies; fa_attention_workspace_size sees that without v
    assert L.fa_attention_workspace_size_qkv(by(q8), by(ki), by(k8), 0) == base + qcopy + kcopy
    assert L.fa_attention_workspace_size(by(q8), by(ki), 0) == base + qcopy + kcopy
    # Q and K alike, only V differs: only the three-branch query knows
    assert L.fa_attention_workspace_size(by(q8), by(k8), 0) == base
    assert L.fa_attention_workspace_size_qkv(by(q8), by(k8), by(vf), 0) == base + qcopy + kcopy
    assert L.fa_attention_workspace_size_qkv(by(q8), by(k8), by(k8), 0) == base
    assert L.fa_attention_workspace_size_qkv(by(q8), by(k8), None, 0) == 0
    # a workspace sized for the uniform call is too small once V differs
    assert L.fa_attention_quant(by(q8), by(k8), by(vf), 0, 0.0, 0x60000, None, 0, 0x70000, base, None) == 7
    # a float branch without data, or with an unsupported head_dim
    qnull = _q(N, 0, B=B, H=Hq, S=Sq, D=D)
    qnull.codes = None
    assert L.fa_attention_quant(by(qnull), by(k8), by(k8), 0, 0.0, 0x60000, None, 0, None, 0, None) == 1
    q96 = _q(N, 0, B=B, H=Hq, S=Sq, D=96)
    assert L.fa_attention_quant(by(q96), by(kf), by(vf), 0, 0.0, 0x60000, None, 0, None, 0, None) == 2
    # an MX V in a mixed call needs head_dim 128
    q64, k64 = _q(N, 2, B=B, H=Hq, S=Sq, D=64), _q(N, 2, B=B, H=Hkv, S=Sk, D=64)
    vm64 = _q(N, 3, B=B, H=Hkv, S=Sk, D=64)
    assert L.fa_attention_quant(by(q64), by(k64), by(vm64), 0, 0.0, 0x60000, None, 0, None, 0, None) == 2
