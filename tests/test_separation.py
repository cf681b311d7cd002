"""The oracle and the CUDA path share no code: the package (Python binding and
CUDA sources) never imports or reads the oracle, and the oracle never imports
the package or loads its library. Only the seeded input generators
(int8_weight_quantized_w4_b200/synth.py, which hold no arithmetic of the
method) serve both, from the test side."""

import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "int8_weight_quantized_w4_b200")


def _sources(pattern):
    return [p for p in glob.glob(pattern, recursive=True) if "/_build/" not in p]


def test_package_never_touches_the_oracle():
    for path in _sources(os.path.join(PKG, "**", "*.py")) + _sources(os.path.join(PKG, "csrc", "*")):
        text = open(path, errors="replace").read()
        assert not re.search(r"^\s*(import|from)\s+oracle\b", text, flags=re.M), path
        assert "oracle/" not in text and "w4_oracle" not in text, path


def test_oracle_never_touches_the_package():
    for path in _sources(os.path.join(ROOT, "oracle", "**", "*.py")):
        text = open(path).read()
        assert "int8_weight_quantized_w4_b200" not in text, path
        assert "libw4b200" not in text and "ctypes" not in text, path


def test_synth_holds_no_method_arithmetic():
    """synth.py draws random numbers and shapes; its code calls nothing that
    packs, dequantises or multiplies matrices."""
    import ast
    tree = ast.parse(open(os.path.join(PKG, "synth.py")).read())
    for node in ast.walk(tree):
        assert not isinstance(node, ast.MatMult), "matrix product in synth.py"
        if isinstance(node, ast.Call):
            f = node.func
            name = f.attr if isinstance(f, ast.Attribute) else getattr(f, "id", "")
            for word in ("dequant", "unpack", "pack", "rint", "matmul", "einsum", "dot", "quantize"):
                assert word not in name.lower(), f"synth.py calls {name}"
