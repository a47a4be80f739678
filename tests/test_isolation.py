"""The product path and the oracle stay apart (CPU): the library fails
loudly when its compiled extension is missing (no CPU fallback), importing
the package and running its layer code never loads the oracle, and neither
side's sources reach into the other's."""
import glob
import os
import re
import subprocess
import sys

import pytest

from mixture_experts_routing_top_b200 import libmoe as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "mixture_experts_routing_top_b200")


def test_missing_extension_fails_loudly(monkeypatch):
    monkeypatch.setattr(M, "SO_PATH", os.path.join(ROOT, "no_such_dir", "libmoe.so"))
    monkeypatch.setattr(M, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        M.lib()


def test_package_import_does_not_load_the_oracle():
    code = ("import sys; import mixture_experts_routing_top_b200.libmoe, mixture_experts_routing_top_b200.layer, "
            "mixture_experts_routing_top_b200.workloads; "
            "print(any(m == 'oracle' or m.startswith('oracle.') for m in sys.modules))")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == "False"


def _sources(root, exts):
    out = []
    for ext in exts:
        out += glob.glob(os.path.join(root, "**", "*" + ext), recursive=True)
    return [p for p in out if "_build" not in p]


def test_product_sources_never_reference_the_oracle():
    for p in _sources(PKG, (".py", ".cu", ".cuh", ".c", ".h")) + _sources(os.path.join(ROOT, "include"), (".h",)):
        text = open(p, encoding="utf-8").read()
        assert not re.search(r"^\s*(from|import)\s+oracle\b", text, re.M), p
        assert "moe_oracle" not in text and "oracle/" not in text, p


def test_oracle_sources_never_reference_the_library():
    for p in _sources(os.path.join(ROOT, "oracle"), (".py", ".c", ".h")):
        text = open(p, encoding="utf-8").read()
        for word in ("libmoe", "csrc", "layer", "cuda", "torch"):
            assert not re.search(r"^\s*(from|import|#include)\b.*\b%s\b" % word, text, re.M), (p, word)
