"""The CUDA library and the oracle share no code (CPU only): no package module
imports the oracle, no kernel source includes it, and nothing under oracle/
imports the package or includes its kernel sources.  Only the seeded input
generators (workloads.py, which holds none of the method's arithmetic) serve
both sides."""
import ast
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "gated_delta_rule_attn_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _files(top, exts):
    for d, _, names in os.walk(top):
        for n in names:
            if n.endswith(exts):
                yield os.path.join(d, n)


def _imported_modules(path):
    tree = ast.parse(open(path, encoding="utf-8").read(), filename=path)
    mods = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            mods.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            mods.add(node.module.split(".")[0])
    return mods


def _includes(path):
    return re.findall(r'#\s*include\s*[<"]([^>"]+)[>"]', open(path, encoding="utf-8", errors="replace").read())


def test_package_never_reaches_the_oracle():
    py = list(_files(PKG, (".py",)))
    assert py
    for f in py:
        assert "oracle" not in _imported_modules(f), f
        src = open(f, encoding="utf-8").read()
        assert not re.search(r"['\"/]oracle[/'\"]", src), f   # no path into oracle/
    for f in _files(os.path.join(PKG, "csrc"), (".cu", ".cuh", ".h", ".cpp")):
        assert not any("oracle" in i or "la_oracle" in i for i in _includes(f)), f


def test_oracle_never_reaches_the_package():
    files = list(_files(ORACLE, (".py",)))
    assert files
    for f in files:
        assert "gated_delta_rule_attn_b200" not in _imported_modules(f), f
    for f in _files(ORACLE, (".c", ".h", ".cpp")):
        assert not any("csrc" in i or i.endswith(".cuh") or i == "la.h" for i in _includes(f)), f


def test_package_fails_loudly_without_its_library(monkeypatch, tmp_path):
    """No CPU fallback: with the CUDA library missing, the first call into the
    package raises instead of computing anything."""
    import pytest
    import gated_delta_rule_attn_b200 as la
    monkeypatch.setattr(la, "_lib", None)
    monkeypatch.setattr(la, "LIB_PATH", str(tmp_path / "libla_b200.so"))
    with pytest.raises(ImportError, match="no CPU fallback"):
        la.lib()
    with pytest.raises(ImportError):
        la.abi_version()
