"""The product path has no CPU fallback: with the CUDA library absent, every entry point of the
binding raises ImportError naming the missing file (checked on the CPU by pointing the loader at
a path that does not exist), and nothing in the package imports the oracle."""
import ast
import pathlib

import numpy as np
import pytest

from recurrent_state_quantization_gated_b200 import _lib, api

PKG = pathlib.Path(_lib.__file__).resolve().parent


@pytest.fixture
def no_library(monkeypatch):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", PKG / "_build_absent" / "libstepq.so")


def test_calls_raise_when_the_library_is_missing(no_library):
    with pytest.raises(ImportError, match="libstepq.so is missing"):
        api.stepq_allocate_bits(np.ones((2, 3)), [4, 6, 8], 12, 1)
    with pytest.raises(ImportError, match="libstepq.so is missing"):
        api.stepq_packed_layout(np.full((2, 64), 6, np.uint8), 64)
    with pytest.raises(ImportError, match="libstepq.so is missing"):
        api.stepq_build_info()


def test_the_package_never_imports_the_oracle():
    for path in PKG.rglob("*.py"):
        tree = ast.parse(path.read_text())
        for node in ast.walk(tree):
            names = []
            if isinstance(node, ast.Import):
                names = [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom):
                names = [node.module or ""]
            assert not any(n == "oracle" or n.startswith("oracle.") for n in names), f"{path} imports the oracle"
