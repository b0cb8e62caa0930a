"""The oracle and the CUDA path stay independent, and the product path has no
fallback.

* No source of the library (csrc/, the binding, the header) mentions the
  oracle, and no oracle source includes or imports the library; the only
  module both sides read is workloads.py, which draws random inputs.
* Without libbitlinear.so the binding raises instead of computing anything.
"""
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "ternary_weight_linear_forward_b200")


def _read(paths):
    return {p: open(p, encoding="utf-8").read() for p in paths}


def test_library_sources_do_not_touch_the_oracle():
    srcs = _read(glob.glob(os.path.join(PKG, "csrc", "*")) + glob.glob(os.path.join(PKG, "*.py")) +
                 [os.path.join(ROOT, "include", "bitlinear.h")])
    for path, text in srcs.items():
        assert not re.search(r"\boracle\b|orc_|liboracle", text), path


def test_oracle_does_not_touch_the_library():
    srcs = _read(glob.glob(os.path.join(ROOT, "oracle", "*.py")) + glob.glob(os.path.join(ROOT, "oracle", "*.c")))
    for path, text in srcs.items():
        assert not re.search(r"bitlinear\.h|libbitlinear|ternary_weight_linear_forward_b200|csrc", text), path


def _code_only(path):
    """The module's code with docstrings and comments dropped."""
    import ast
    tree = ast.parse(open(path, encoding="utf-8").read())
    for node in ast.walk(tree):
        body = getattr(node, "body", None)
        if isinstance(body, list) and body and isinstance(body[0], ast.Expr) and \
                isinstance(getattr(body[0], "value", None), ast.Constant) and isinstance(body[0].value.value, str):
            body.pop(0)
    return ast.unparse(tree)


def test_shared_input_module_holds_no_method_arithmetic():
    code = _code_only(os.path.join(ROOT, "workloads.py"))
    assert "oracle" not in code and "ternary_weight_linear_forward_b200" not in code
    # no quantiser, ternariser or packing: no 127 / rint / clip, no absmean
    # (byte counts such as packed_bytes are bookkeeping for the roofline)
    for pat in (r"absmean", r"\brint\b", r"\b127\b", r"\bclip\b", r"ternar", r"\bpack\s*\("):
        assert not re.search(pat, code), pat


def test_binding_fails_loudly_without_the_library(monkeypatch):
    from ternary_weight_linear_forward_b200 import bitlinear as B
    monkeypatch.setattr(B, "LIB_PATH", os.path.join(PKG, "no_such_libbitlinear.so"))
    monkeypatch.setattr(B, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        B.lib()
