"""Static checks that the CUDA product path and the fp64 oracle stay apart: the package never
imports or links the oracle, the oracle never uses the package's kernels or headers, bench.py
imports the oracle only inside its CPU-baseline and reference-arm functions, and the binding
fails loudly (no fallback) when libgdn.so is missing."""
import ast
import os
import re

import pytest

import gated_deltanet_layer_02_b200 as gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "gated_deltanet_layer_02_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _sources(top, exts):
    for dirpath, dirnames, files in os.walk(top):
        dirnames[:] = [d for d in dirnames if not d.startswith(("_build", "__pycache__"))]
        for f in files:
            if f.endswith(exts):
                yield os.path.join(dirpath, f)


def test_package_never_uses_the_oracle():
    pat = re.compile(r"^\s*(import\s+oracle|from\s+oracle\b)|gdn_oracle|liboracle|orc_", re.M)
    hits = [p for p in _sources(PKG, (".py", ".cu", ".cuh", ".h", ".cpp"))
            if pat.search(open(p).read())]
    assert hits == []


def test_oracle_never_uses_the_package():
    pat = re.compile(r"^\s*(import|from)\s+gated_deltanet_layer_02_b200|libgdn\.so|"
                     r"#include\s+\"(gdn|args|tc|common)\.", re.M)
    hits = [p for p in _sources(ORACLE, (".py", ".c", ".h")) if pat.search(open(p).read())]
    assert hits == []


def test_bench_imports_the_oracle_only_in_its_cpu_arms():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    for node in tree.body:   # module level: no oracle import
        if isinstance(node, (ast.Import, ast.ImportFrom)):
            names = [a.name for a in node.names] + [getattr(node, "module", None) or ""]
            assert "oracle" not in names
    users = set()
    for fn in ast.walk(tree):
        if isinstance(fn, ast.FunctionDef):
            for node in ast.walk(fn):
                if isinstance(node, ast.Import) and any(a.name == "oracle" for a in node.names):
                    users.add(fn.name)
    assert users == {"cpu_oracle_rate", "run_reference"}, users


def test_binding_raises_without_the_library(monkeypatch):
    monkeypatch.setattr(gdn, "_lib", None)
    monkeypatch.setattr(gdn, "LIB_PATH", os.path.join(ROOT, "no_such_dir", "libgdn.so"))
    with pytest.raises(RuntimeError, match="missing"):
        gdn.lib()
