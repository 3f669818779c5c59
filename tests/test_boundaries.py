"""Structural rules of the repository, checked on the host: the product
package never reaches the oracle, the oracle never reaches the CUDA path,
and the CUDA sources carry no CPU arithmetic fallback."""

import ast
import glob
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _imports(path):
    tree = ast.parse(open(path).read())
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module:
            names.add(node.module.split(".")[0])
    return names


def test_product_package_never_imports_the_oracle():
    for path in glob.glob(os.path.join(ROOT, "sparse_key_value_b200", "*.py")):
        assert "oracle" not in _imports(path), path


def test_oracle_never_imports_the_product_package():
    for path in glob.glob(os.path.join(ROOT, "oracle", "*.py")):
        assert "sparse_key_value_b200" not in _imports(path), path
    src = open(os.path.join(ROOT, "oracle", "pkm_oracle.c")).read()
    assert "pkm.h" not in src and "csrc" not in src


def test_cuda_sources_do_not_include_the_oracle():
    for path in glob.glob(os.path.join(ROOT, "sparse_key_value_b200", "csrc", "*")):
        src = open(path).read()
        assert "oracle" not in src.lower(), path


def test_binding_fails_loudly_without_the_library(tmp_path):
    """The binding raises when libpkm.so is missing: there is no fallback."""
    import pytest

    from sparse_key_value_b200 import _lib

    with pytest.raises(ImportError):
        _lib.load(str(tmp_path / "missing_libpkm.so"))
