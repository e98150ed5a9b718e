"""The product path and the oracle stay apart (no GPU needed).

The CUDA path (the package, its CUDA sources and libfaq.so) must never reach
the oracle, and the oracle must never reach the CUDA path; the input
generators that both use import neither.  The binding must fail loudly when
libfaq.so is missing instead of falling back to anything else.
"""
import ast
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "quantized_attention_amax_b200")


def files(top, exts):
    for d, subdirs, names in os.walk(top):
        subdirs[:] = [s for s in subdirs if not s.startswith(("_build", "__pycache__"))]
        for n in names:
            if n.endswith(exts):
                yield os.path.join(d, n)


def imported_modules(path):
    tree = ast.parse(open(path).read(), path)
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield a.name.split(".")[0]
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            yield node.module.split(".")[0]


def test_package_never_imports_the_oracle():
    for f in files(PKG, (".py",)):
        assert "oracle" not in set(imported_modules(f)), f


def test_cuda_sources_never_name_the_oracle():
    for f in files(PKG, (".cu", ".cuh", ".h")):
        text = open(f).read()
        assert "faq_oracle" not in text and not re.search(r"\borc_\w+\s*\(", text), f


def test_oracle_never_reaches_the_cuda_path():
    for f in files(os.path.join(ROOT, "oracle"), (".py",)):
        assert "quantized_attention_amax_b200" not in set(imported_modules(f)), f
    for f in files(os.path.join(ROOT, "oracle"), (".c", ".h")):
        text = open(f).read()
        assert not re.search(r'#include\s+"(faq\.h|sm100|internal|quant_common|attn_common)', text), f


def test_input_generators_import_neither_side():
    for f in files(os.path.join(ROOT, "workloads"), (".py",)):
        mods = set(imported_modules(f))
        assert "oracle" not in mods and "quantized_attention_amax_b200" not in mods, f


def needed(lib):
    out = subprocess.run(["readelf", "-d", lib], capture_output=True, text=True).stdout
    return re.findall(r"\(NEEDED\)\s+Shared library: \[([^\]]+)\]", out)


def test_libraries_do_not_link_each_other():
    from oracle import build as ob
    from quantized_attention_amax_b200 import build as pb
    lib_faq, lib_orc = pb.build(), ob.build()
    assert not any("oracle" in n for n in needed(lib_faq))
    assert not any("faq" in n for n in needed(lib_orc))


def test_binding_raises_without_the_library(monkeypatch, tmp_path):
    from quantized_attention_amax_b200 import _native
    monkeypatch.setattr(_native, "LIB_PATH", str(tmp_path / "libfaq.so"))
    monkeypatch.setattr(_native, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        _native.lib()
