"""The product path has no CPU fallback and never reaches the oracle: a missing libcowa.so makes
every call raise, CPU tensors are refused before any library call, and no module of the package
imports anything from oracle/ (checked on the source)."""

import ast
import os

import pytest
import torch

from structured_sparse_attention_cowa_b200 import cowa as cw

PKG = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "structured_sparse_attention_cowa_b200")


def test_missing_library_raises(monkeypatch):
    monkeypatch.setattr(cw, "_lib", None)
    monkeypatch.setattr(cw, "LIB_PATH", os.path.join(PKG, "no_such_libcowa.so"))
    with pytest.raises(RuntimeError, match="libcowa.so not found"):
        cw.lib()
    with pytest.raises(RuntimeError):
        cw.visible_counts(cw.Pattern(4, 8, 64, 1), 1, 64)


def test_cpu_tensors_are_refused():
    pat = cw.Pattern(4, 8, 64, 2)
    q = torch.zeros((1, 64, 4, 64), dtype=torch.bfloat16)
    k = torch.zeros((1, 64, 2, 64), dtype=torch.bfloat16)
    lse = torch.zeros((1, 4, 64))
    with pytest.raises(TypeError):
        cw.cowa_fwd(q, k, k, pat)
    with pytest.raises(TypeError):
        cw.cowa_bwd(q, k, k, q, lse, q, pat)
    with pytest.raises(TypeError):
        cw.cowa_bwd_varlen(q[0], k[0], k[0], q[0], lse[0], q[0], [0, 64], pat)
    with pytest.raises(TypeError):
        cw.cowa_fwd(q.float(), k, k, pat)


def test_package_never_imports_the_oracle():
    for name in sorted(os.listdir(PKG)):
        if not name.endswith(".py"):
            continue
        tree = ast.parse(open(os.path.join(PKG, name)).read())
        for node in ast.walk(tree):
            if isinstance(node, ast.Import):
                assert not any(a.name.split(".")[0] == "oracle" for a in node.names), name
            elif isinstance(node, ast.ImportFrom):
                assert (node.module or "").split(".")[0] != "oracle", name
    for name in sorted(os.listdir(os.path.join(PKG, "csrc"))):
        src = open(os.path.join(PKG, "csrc", name), errors="replace").read()
        assert "oracle" not in src.lower() or name.endswith(".py"), name
