"""The product path has no fallback: without libdory.so the binding raises
instead of computing anything, and no module of the package reaches the
oracle (CPU only)."""
import ast
import os

import pytest

import looped_ngpt_b200 as lb
from looped_ngpt_b200 import _lib

PKG = os.path.dirname(os.path.abspath(lb.__file__))


def test_missing_library_raises(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libdory.so"))
    with pytest.raises(RuntimeError, match="missing"):
        _lib.load()


def _imported_modules(path):
    tree = ast.parse(open(path).read(), filename=path)
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield a.name
        elif isinstance(node, ast.ImportFrom) and node.module:
            yield node.module


def test_package_never_imports_the_oracle():
    files = [os.path.join(PKG, f) for f in os.listdir(PKG) if f.endswith(".py")]
    assert files
    for f in files:
        for mod in _imported_modules(f):
            assert not mod.split(".")[0] == "oracle", (f, mod)
