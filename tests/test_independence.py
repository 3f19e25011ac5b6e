"""The oracle and the CUDA path stay independent, and the product path has no
fallback: checked on the sources, with no GPU.

- Nothing in the package (Python, CUDA, the build) imports, includes, links
  or loads anything under oracle/, and the oracle uses nothing of the
  package.
- bench.py touches the oracle only in its CPU-baseline legs.
- Without libsmla.so every binding call raises.
"""
import ast
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sparse_mla_decode_partial_b200")
ORACLE = os.path.join(ROOT, "oracle")


def source_files(top, exts):
    for d, _, files in os.walk(top):
        for f in files:
            if f.endswith(exts):
                yield os.path.join(d, f)


def code_only(text, ext):
    """The text without comments and docstrings (a comment may name the
    other side; code may not use it)."""
    if ext == ".py":
        tree = ast.parse(text)
        names = []
        for node in ast.walk(tree):
            if isinstance(node, ast.Import):
                names += [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom):
                names.append(node.module or "")
            elif isinstance(node, ast.Constant) and isinstance(node.value, str):
                continue
            elif isinstance(node, ast.Name):
                names.append(node.id)
            elif isinstance(node, ast.Attribute):
                names.append(node.attr)
        return " ".join(names)
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    return re.sub(r"//[^\n]*", " ", text)


def test_package_uses_nothing_of_the_oracle():
    for path in source_files(PKG, (".py", ".cu", ".cuh", ".h")):
        code = code_only(open(path).read(), os.path.splitext(path)[1])
        assert not re.search(r"\boracle\b|smla_oracle|smla_indexer_oracle", code), path
    build_src = open(os.path.join(PKG, "build.py")).read()
    assert "oracle" not in code_only(build_src, ".py")


def test_oracle_uses_nothing_of_the_package():
    for path in source_files(ORACLE, (".py", ".c", ".h")):
        ext = os.path.splitext(path)[1]
        text = open(path).read()
        code = code_only(text, ext)
        assert "sparse_mla_decode_partial_b200" not in code, path
        assert not re.search(r"\bcsrc\b|smla\.h|libsmla\.so|binding", code), path
        if ext == ".c":
            for inc in re.findall(r'#include\s*[<"]([^>"]+)[>"]', code):
                assert "/" not in inc and not inc.startswith("smla"), (path, inc)


def test_bench_touches_the_oracle_only_in_its_cpu_legs():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    allowed = {"cpu_baseline", "indexer_cpu_baseline"}

    def visit(node, func):
        for child in ast.iter_child_nodes(node):
            f = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else func
            if isinstance(child, ast.Import):
                for a in child.names:
                    if a.name.split(".")[0] == "oracle":
                        assert f in allowed, (f, a.name)
            elif isinstance(child, ast.ImportFrom) and (child.module or "").split(".")[0] == "oracle":
                assert f in allowed, (f, child.module)
            visit(child, f)
    visit(tree, None)


def test_binding_raises_without_the_library(monkeypatch, tmp_path):
    from sparse_mla_decode_partial_b200 import binding
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "libsmla.so"))
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(RuntimeError, match="is missing"):
        binding.lib()
    with pytest.raises(RuntimeError, match="is missing"):
        binding.choose_nsplit(1, 1, 16, 2048, 148)
