"""The oracle's pins catch planted mistakes.

Each case below copies oracle/faq_oracle.c, plants one plausible mistake in
the copy (a wrong rounding rule, a dropped term, a wrong index, a transposed
operand, a wrong constant), compiles it the way oracle/build.py compiles the
oracle, and runs every pin of the oracle's test modules against it.  The
case passes when at least one pin fails.  A control compiles the unmodified
source the same way and checks that every pin passes, so a failure here
means the pins are too weak for that mistake, not that the harness is broken.

The mistakes are planted on the CPU in a private copy; neither the oracle nor
anything on the GPU path is touched.
"""
import concurrent.futures
import inspect
import os
import subprocess

import pytest

import oracle
from oracle import build as oracle_build

import test_oracle_attention
import test_oracle_codecs
import test_oracle_modes_next
import test_oracle_quant

# cheapest first: the exhaustive codec sweeps take most of the time
PIN_MODULES = [test_oracle_attention, test_oracle_quant, test_oracle_modes_next, test_oracle_codecs]

# (name, function whose body holds the mistake, original text, planted text)
MUTANTS = [
    ("e4m3 ties away from zero", "uint8_t orc_e4m3_encode(",
     "double r = rint(a / quantum) * quantum;", "double r = floor(a / quantum + 0.5) * quantum;"),
    ("e4m3 without saturation", "uint8_t orc_e4m3_encode(", "if (r > 448.0) r = 448.0;", ";"),
    ("e4m3 subnormal spacing 2^-10", "uint8_t orc_e4m3_encode(", "quantum = 0x1p-9;", "quantum = 0x1p-10;"),
    ("e2m1 spacing 0.5 in [2, 4)", "uint8_t orc_e2m1_encode(", "quantum = 1.0;", "quantum = 0.5;"),
    ("int8 clamp to -127", "int8_t orc_int8_encode(", "if (r < -128.0) r = -128.0;",
     "if (r < -127.0) r = -127.0;"),
    ("int8 truncation", "int8_t orc_int8_encode(", "double r = rint((double)v);", "double r = trunc((double)v);"),
    ("mx exponent one too high", "int orc_mx_exponent(float", "int x = (e - 1) - 2;", "int x = e - 2;"),
    ("mxfp8 exponent with e2m1's emax", "int orc_mx_exponent_e4m3(", "int x = (e - 1) - 8;",
     "int x = (e - 1) - 2;"),
    ("bf16 with 9 significant bits", "uint16_t orc_f64_to_bf16(", "quantum = ldexp(1.0, e - 8);",
     "quantum = ldexp(1.0, e - 9);"),
    ("calibration forgets earlier batches", "void orc_calibrate_per_head(", "float m = amax[h];",
     "float m = 0.0f;"),
    ("int8 per-head scale amax / 128", "void orc_quantize_int8_per_head(", "amax[h] / 127.0f",
     "amax[h] / 128.0f"),
    ("fp8 per-token amax misses the last channel", "void orc_quantize_fp8_per_token(",
     "for (int d = 0; d < D; ++d) {", "for (int d = 0; d < D - 1; ++d) {"),
    ("fp8 per-token scales indexed [h, b, s]", "void orc_quantize_fp8_per_token(",
     "scales[((size_t)b * H + h) * S + s] = sc;", "scales[((size_t)h * B + b) * S + s] = sc;"),
    ("fp8 per-head scale amax / 127", "void orc_quantize_fp8_per_head(", "amax[h] / 448.0f", "amax[h] / 127.0f"),
    ("int8 per-token scale amax / 448", "void orc_quantize_int8_per_token(", "amax / 127.0f", "amax / 448.0f"),
    ("mxfp4 nibbles swapped", "void orc_quantize_mxfp4(", "(uint8_t)(lo | (hi << 4))", "(uint8_t)(hi | (lo << 4))"),
    ("fp8 block amax from its first token", "void orc_quantize_fp8_block(",
     "for (int s = s0; s < s1; ++s)\n          for (int d = 0; d < D; ++d) {\n            const float a",
     "for (int s = s0; s < s0 + 1; ++s)\n          for (int d = 0; d < D; ++d) {\n            const float a"),
    ("rotation by R transposed", "void orc_rotate_f64(", "R[(size_t)d * D + j]", "R[(size_t)j * D + d]"),
    ("int8 per-token dequantized with a per-head scale", "case ORC_MODE_INT8_PER_TOKEN:",
     "((const float*)t->scales)[((size_t)b * t->H + h) * t->S + s]", "((const float*)t->scales)[h]"),
    ("mxfp4 dequant nibble order", "case ORC_MODE_MXFP4:",
     "(d & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15)",
     "(d & 1) ? (uint8_t)(byte & 15) : (uint8_t)(byte >> 4)"),
    ("softmax scale 1 / D", "void orc_attention(", "scale = 1.0 / sqrt((double)D);", "scale = 1.0 / (double)D;"),
    ("causal mask aligned top-left", "void orc_attention(", "const int last = causal ? i + (Sk - Sq) : Sk - 1;",
     "const int last = causal ? i : Sk - 1;"),
    ("GQA query heads interleaved", "void orc_attention(", "const int h = hk * group + g;",
     "const int h = g * Hkv + hk;"),
    ("QK^T drops the last channel", "void orc_attention(",
     "for (int d = 0; d < D; ++d) acc += qr[d]", "for (int d = 0; d < D - 1; ++d) acc += qr[d]"),
    ("softmax sum without the last key", "void orc_attention(", "l += sc[j];", "if (j + 1 < nvis) l += sc[j];"),
    ("P V multiplies K", "void orc_attention(", "const double* vr = vd + (size_t)j * D;",
     "const double* vr = kd + (size_t)j * D;"),
    ("lse without the log", "void orc_attention(", "m + log(l)", "m + l"),
    ("int8 per-token amax misses the last channel", "void orc_quantize_int8_per_token(",
     "for (int d = 0; d < D; ++d) {", "for (int d = 0; d < D - 1; ++d) {"),
    ("mxfp4 block amax misses its last element", "void orc_quantize_mxfp4(", "for (int j = 0; j < 32; ++j) {",
     "for (int j = 0; j < 31; ++j) {"),
    ("mxfp8 block amax misses its last element", "void orc_quantize_mxfp8(", "for (int j = 0; j < 32; ++j) {",
     "for (int j = 0; j < 31; ++j) {"),
    ("calibration skips the last token", "void orc_calibrate_per_head(", "for (int s = 0; s < S; ++s)",
     "for (int s = 0; s < S - 1; ++s)"),
    ("BSND read as BNSD", "static size_t elem_index(", "return (((size_t)b * S + s) * H + h) * D + d;",
     "return (((size_t)b * H + h) * S + s) * D + d;"),
    ("e4m3 decode subnormals at 2^-10", "double orc_e4m3_decode(", "ldexp((double)m, -9)",
     "ldexp((double)m, -10)"),
    ("e2m1 decode top value 8", "double orc_e2m1_decode(", "4.0, 6.0}", "4.0, 8.0}"),
    ("fp8 per-token dequantized with [h, b, s] scales", "case ORC_MODE_FP8_PER_TOKEN:",
     "((const float*)t->scales)[((size_t)b * t->H + h) * t->S + s]",
     "((const float*)t->scales)[((size_t)h * t->B + b) * t->S + s]"),
    ("fp8 block scales indexed [h, b, g]", "void orc_quantize_fp8_block(",
     "scales[((size_t)b * H + h) * nblk + g] = sc;", "scales[((size_t)h * B + b) * nblk + g] = sc;"),
    ("mxfp4 scales indexed [h, b, s]", "void orc_quantize_mxfp4(", "e8m0[(((size_t)b * H + h) * S + s) * G + g]",
     "e8m0[(((size_t)h * B + b) * S + s) * G + g]"),
    ("mxfp8 scales indexed [h, b, s]", "void orc_quantize_mxfp8(", "e8m0[(((size_t)b * H + h) * S + s) * G + g]",
     "e8m0[(((size_t)h * B + b) * S + s) * G + g]"),
    ("rotation rounded to bf16 through fp32", "void orc_rotate(const", "out[i] = orc_f64_to_bf16(tmp[i]);",
     "out[i] = orc_f64_to_bf16((double)(float)tmp[i]);"),
    ("e4m3 exponent bias 8", "uint8_t orc_e4m3_encode(", "((E + 7) << 3)", "((E + 8) << 3)"),
    ("e8m0 byte e + 128", "void orc_quantize_mxfp4(", "(uint8_t)(e + 127)", "(uint8_t)(e + 128)"),
    ("zero fp8 scale divides anyway", "void orc_quantize_fp8_per_token(",
     "(sc > 0.0f) ? orc_e4m3_encode(xf / sc) : (uint8_t)0", "orc_e4m3_encode(xf / sc)"),
    ("causal mask one key short", "void orc_attention(", "const int last = causal ? i + (Sk - Sq) : Sk - 1;",
     "const int last = causal ? i + (Sk - Sq) - 1 : Sk - 1;"),
    ("a row with no visible key divides by zero", "void orc_attention(", "if (nvis <= 0) {", "if (nvis < 0) {"),
    ("sampled rows ignored", "void orc_attention(", "const int i = rows ? rows[r] : r;", "const int i = r;"),
    ("fp8 per-head dequantized with head 0's scale", "case ORC_MODE_FP8_PER_HEAD:", "((const float*)t->scales)[h]",
     "((const float*)t->scales)[0]"),
    ("int8 per-head dequantized with head 0's scale", "case ORC_MODE_INT8_PER_HEAD:", "((const float*)t->scales)[h]",
     "((const float*)t->scales)[0]"),
    ("mxfp8 dequant exponent bias 128", "case ORC_MODE_MXFP8: {", "- 127;", "- 128;"),
    ("fp8 block dequantized with the next block's scale", "case ORC_MODE_FP8_BLOCK: {", "nblk + s / t->blk]",
     "nblk + (s / t->blk + 1) % nblk]"),
    ("float branch reads the neighbouring element", "case ORC_MODE_FLOAT:", "((const uint16_t*)t->codes)[i]",
     "((const uint16_t*)t->codes)[i ^ 1]"),
    ("bf16 overflow saturates instead of rounding to infinity", "uint16_t orc_f64_to_bf16(", "bits = 0x7F80;",
     "bits = 0x7F7F;"),
    ("e4m3 NaN encoded as 448", "uint8_t orc_e4m3_encode(", "if (isnan(v)) return 0x7F;", "if (isnan(v)) return 0x7E;"),
    ("e2m1 infinity encoded as 0", "uint8_t orc_e2m1_encode(", "if (isnan(a) || isinf(a)) a = 6.0;",
     "if (isnan(a) || isinf(a)) a = 0.0;"),
    ("int8 NaN encoded as 127", "int8_t orc_int8_encode(", "if (isnan(v)) return 0;", "if (isnan(v)) return 127;"),
    ("calibration without the absolute value", "void orc_calibrate_per_head(",
     "const float a = fabsf(orc_bf16_to_f32(", "const float a = (orc_bf16_to_f32("),
    ("e4m3 sign dropped", "uint8_t orc_e4m3_encode(", "return (uint8_t)(code | (neg ? 0x80u : 0u));",
     "return (uint8_t)code;"),
    ("e2m1 loses the sign of -0", "uint8_t orc_e2m1_encode(", "const int neg = signbit(v) ? 1 : 0;",
     "const int neg = v < 0.0f ? 1 : 0;"),
    ("rotation accumulated in fp32", "void orc_rotate_f64(", "double acc = 0.0;", "float acc = 0.0f;"),
    ("caller's softmax scale ignored", "void orc_attention(", "if (scale <= 0.0) scale = 1.0 / sqrt((double)D);",
     "scale = 1.0 / sqrt((double)D);"),
    ("lse written to the mirrored row", "void orc_attention(",
     "lse[((size_t)b * Hq + h) * nrows + r] = m + log(l);", "lse[((size_t)b * Hq + h) * nrows + (nrows - 1 - r)] = m + log(l);"),
    ("calibration reads the first batch entry only", "void orc_calibrate_per_head(", "for (int b = 0; b < B; ++b)",
     "for (int b = 0; b < 1; ++b)"),
    ("mxfp4 odd elements coded from the even one", "void orc_quantize_mxfp4(",
     "x[elem_index(layout, H, S, D, b, h, s, d + 1)]", "x[elem_index(layout, H, S, D, b, h, s, d)]"),
]


def plant(src: str, anchor: str, old: str, new: str) -> str:
    at = src.index(anchor)
    i = src.index(old, at)
    return src[:i] + new + src[i + len(old):]


def compile_copy(text: str, path: str) -> str:
    c = path[:-3] + ".c"
    with open(c, "w") as f:
        f.write(text)
    # the flags of oracle/build.py, with the header found beside the original source
    subprocess.check_call(["gcc", "-std=c99", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC",
                           "-shared", "-w", "-I", oracle_build.HERE, "-o", path, c, "-lm"])
    return path


def pins():
    """(label, call) for every pin that reads the oracle, parametrized cases expanded."""
    out = []
    for mod in PIN_MODULES:
        for name, fn in sorted(inspect.getmembers(mod, inspect.isfunction), key=lambda kv: kv[1].__code__.co_firstlineno):
            if not name.startswith("test_") or fn.__module__ != mod.__name__:
                continue
            params = list(inspect.signature(fn).parameters)
            if "orc" not in params:
                continue
            cases = [{}]
            for m in getattr(fn, "pytestmark", []):
                if m.name == "parametrize":
                    names = [s.strip() for s in m.args[0].split(",")] if isinstance(m.args[0], str) else list(m.args[0])
                    cases = [dict(c, **dict(zip(names, v if len(names) > 1 else (v,)))) for c in cases
                             for v in m.args[1]]
            for c in cases:
                out.append((f"{mod.__name__}.{name}{c or ''}", lambda fn=fn, c=c: fn(oracle, **c)))
    return out


@pytest.fixture(scope="module")
def libs(tmp_path_factory):
    d = tmp_path_factory.mktemp("oracle_mutants")
    src = open(oracle_build.SRC).read()
    jobs = {"control": src}
    for name, anchor, old, new in MUTANTS:
        jobs[name] = plant(src, anchor, old, new)
    with concurrent.futures.ThreadPoolExecutor(max_workers=8) as ex:
        futs = {k: ex.submit(compile_copy, t, str(d / f"m{i}.so")) for i, (k, t) in enumerate(jobs.items())}
        return {k: f.result() for k, f in futs.items()}


def run_pins_on(path, monkeypatch):
    """Load the compiled copy as the oracle's library and run the pins; returns the first failing pin."""
    monkeypatch.setattr(oracle_build, "build", lambda force=False: path)
    monkeypatch.setattr(oracle, "_lib", None)
    oracle.lib()
    for label, call in pins():
        try:
            call()
        except Exception as e:  # an assertion, or numpy refusing a malformed result
            return f"{label}: {type(e).__name__}"
    return None


def test_control_copy_passes_every_pin(libs, monkeypatch):
    assert len(pins()) > 40
    assert run_pins_on(libs["control"], monkeypatch) is None


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(libs, monkeypatch, name):
    caught = run_pins_on(libs[name], monkeypatch)
    assert caught is not None, f"no pin fails when the oracle has this mistake: {name}"
