"""The oracle and the CUDA path share no code, and the product path has no CPU fallback.  CPU only.

* No file of the package (Python, CUDA, headers) refers to the oracle, and no file of the oracle
  refers to the package or its CUDA sources; the only module both use is the seeded input
  generator, which holds no arithmetic of the method.
* Only the tests, ``__graft_entry__`` (build, smoke) and ``bench.py`` (its CPU legs) import the
  oracle.
* The tensor-level calls refuse CPU tensors, and a missing library makes loading fail loudly.
"""
import ast
import os
import subprocess
import sys

import pytest
import torch

import causal_sliding_window_swa_b200 as swa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "causal_sliding_window_swa_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _files(top, exts):
    for dirpath, _, names in os.walk(top):
        for n in names:
            if n.endswith(exts):
                yield os.path.join(dirpath, n)


def _imports(path):
    tree = ast.parse(open(path).read())
    out = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            out |= {a.name.split(".")[0] for a in node.names}
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            out.add(node.module.split(".")[0])
    return out


def test_package_never_refers_to_the_oracle():
    for f in _files(PKG, (".py",)):
        assert "oracle" not in _imports(f), f
    for f in _files(PKG, (".cu", ".cuh", ".h")):
        src = open(f).read()
        assert "swa_oracle" not in src and "oracle/" not in src, f
    for f in _files(os.path.join(ROOT, "include"), (".h",)):
        assert "swa_oracle" not in open(f).read(), f


def test_oracle_never_refers_to_the_package():
    for f in _files(ORACLE, (".py",)):
        assert "causal_sliding_window_swa_b200" not in _imports(f), f
    for f in _files(ORACLE, (".c", ".h")):
        src = open(f).read()
        assert "csrc" not in src and "swa_attn.h" not in src and "#include \"" not in src, f


def test_only_tests_entry_and_bench_import_the_oracle():
    allowed = {os.path.join(ROOT, "__graft_entry__.py"), os.path.join(ROOT, "bench.py")}
    for f in _files(ROOT, (".py",)):
        rel = os.path.relpath(f, ROOT)
        if rel.startswith(("tests", "oracle", "_work", ".", "baseline", "build")) or f in allowed:
            continue
        assert "oracle" not in _imports(f), rel


def test_tensor_calls_refuse_cpu_tensors():
    q = torch.zeros((1, 4, 1, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        swa.forward(q, q, q, 0)
    with pytest.raises(ValueError):
        swa.backward(q, q, q, q, torch.zeros((1, 1, 4)), q, 0)


def test_missing_library_fails_loudly():
    code = ("import causal_sliding_window_swa_b200 as swa\n"
            "swa.LIB_PATH = '/nonexistent/libswa_attn.so'\n"
            "try:\n    swa.load()\nexcept (ImportError, OSError):\n    print('raised')\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert "raised" in r.stdout, r.stdout + r.stderr
