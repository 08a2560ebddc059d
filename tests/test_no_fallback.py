"""The product path has no CPU fallback: the binding refuses to import without the built
library, and nothing in the package reaches the oracle."""
import ast
import importlib.util
import os
import shutil

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "longlora_shifted_sparse_b200")


def test_binding_raises_when_library_is_missing(tmp_path):
    d = tmp_path / "pkg"
    d.mkdir()
    shutil.copy(os.path.join(PKG, "s2attn.py"), d / "s2attn.py")   # no libs2attn.so beside it
    spec = importlib.util.spec_from_file_location("s2attn_without_lib", d / "s2attn.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError, match="not built"):
        spec.loader.exec_module(mod)


def _imported_modules(path):
    tree = ast.parse(open(path).read(), filename=path)
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield a.name
        elif isinstance(node, ast.ImportFrom):
            yield node.module or ""


def test_package_never_imports_the_oracle_or_numerics_libraries():
    banned = ("oracle", "synth", "numpy", "scipy", "torch.nn.functional")
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith(".py"):
                path = os.path.join(dirpath, f)
                for m in _imported_modules(path):
                    assert not any(m == b or m.startswith(b + ".") for b in banned), (path, m)


def test_native_sources_do_not_reference_the_oracle():
    for dirpath, _, files in os.walk(os.path.join(PKG, "csrc")):
        for f in files:
            text = open(os.path.join(dirpath, f), errors="replace").read()
            assert "oracle" not in text.lower(), f
