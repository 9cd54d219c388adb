"""CPU checks that the product path and the oracle stay apart: nothing in the
library package or its C/CUDA sources imports, includes or loads the oracle,
the oracle shares no source with the library, and the binding raises when the
compiled library is missing instead of computing anything on the host."""
import ast
import os
import re

import pytest

import rope_context_extension_jet_b200 as jl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "rope_context_extension_jet_b200")


def _files(top, exts):
    for d, _, names in os.walk(top):
        for n in names:
            if n.endswith(exts):
                yield os.path.join(d, n)


def test_package_python_never_imports_the_oracle():
    for path in _files(PKG, (".py",)):
        tree = ast.parse(open(path).read())
        for node in ast.walk(tree):
            if isinstance(node, ast.Import):
                names = [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom):
                names = [node.module or ""]
            else:
                continue
            assert not any(n.split(".")[0] == "oracle" for n in names), path


def test_cuda_sources_never_include_or_load_the_oracle():
    for path in _files(os.path.join(PKG, "csrc"), (".cu", ".cuh", ".h")):
        src = open(path).read()
        assert not re.search(r'#\s*include\s*[<"][^>"]*oracle', src), path
        assert "jetlong_oracle" not in src and "jlo_" not in src, path


def test_oracle_source_shares_nothing_with_the_library():
    src = open(os.path.join(ROOT, "oracle", "jetlong_oracle.c")).read()
    assert not re.search(r'#\s*include\s*"', src)  # system headers only
    for py in _files(os.path.join(ROOT, "oracle"), (".py",)):
        tree = ast.parse(open(py).read())
        for node in ast.walk(tree):
            if isinstance(node, ast.ImportFrom):
                assert not (node.module or "").startswith("rope_context_extension_jet_b200"), py
            if isinstance(node, ast.Import):
                assert not any(a.name.startswith("rope_context_extension_jet_b200") for a in node.names), py


def test_missing_library_raises(tmp_path):
    with pytest.raises(RuntimeError, match="missing"):
        jl.load_library(str(tmp_path / "libjetlong.so"))
