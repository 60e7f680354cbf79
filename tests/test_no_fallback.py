"""The product path has no fallback: the binding fails loudly without libmrf.so, and nothing in
the package reaches the oracle (the oracle is test infrastructure)."""
import ast
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "axial_band_split_b200")


def test_binding_raises_without_the_library(monkeypatch):
    from axial_band_split_b200 import mrf
    monkeypatch.setattr(mrf, "_lib", None)
    monkeypatch.setattr(mrf, "_LIB_PATH", os.path.join(ROOT, "no_such_dir", "libmrf.so"))
    with pytest.raises(ImportError):
        mrf.lib()
    with pytest.raises(ImportError):
        mrf.band_tables(__import__("synth").TINY)


def _imports(path):
    tree = ast.parse(open(path).read(), filename=path)
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield a.name
        elif isinstance(node, ast.ImportFrom):
            yield node.module or ""


def test_package_never_imports_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith(".py"):
                p = os.path.join(dirpath, f)
                for name in _imports(p):
                    assert not name.split(".")[0] == "oracle", f"{p} imports {name}"


def test_native_sources_never_include_the_oracle():
    for dirpath, _, files in os.walk(os.path.join(PKG, "csrc")):
        for f in files:
            src = open(os.path.join(dirpath, f), errors="replace").read()
            assert "oracle/" not in src and "oracle.h" not in src, f
