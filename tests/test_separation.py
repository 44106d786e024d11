"""The oracle and the product share no code, and the product has no CPU path.

* importing the product and loading its library brings in no oracle module;
* no product source names the oracle, and no oracle source names the product
  or includes one of its headers;
* without the built library every compute entry point raises: there is no
  fallback.
"""
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "selective_state_space_momentum_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _files(top, exts):
    for d, _, names in os.walk(top):
        if "_build" in d or "__pycache__" in d:
            continue
        for n in names:
            if n.endswith(exts):
                yield os.path.join(d, n)


def test_product_import_loads_no_oracle():
    code = ("import sys, selective_state_space_momentum_b200 as mm; mm.load_library(); "
            "print(sorted(m for m in sys.modules if m == 'oracle' or m.startswith('oracle.')))")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT, timeout=120)
    assert r.returncode == 0, r.stderr[-1000:]
    assert r.stdout.strip() == "[]"


def test_product_sources_never_name_the_oracle():
    pat = re.compile(r"\bimport\s+oracle\b|\bfrom\s+oracle\b|mm_oracle|liboracle")
    for f in _files(PKG, (".py", ".cu", ".cuh", ".cpp", ".h")):
        with open(f) as fh:
            assert not pat.search(fh.read()), f
    for f in _files(os.path.join(ROOT, "include"), (".h",)):
        with open(f) as fh:
            assert not pat.search(fh.read()), f


def test_oracle_sources_never_name_the_product():
    for f in _files(ORACLE, (".py", ".c", ".h")):
        with open(f) as fh:
            src = fh.read()
        assert not re.search(r"\b(import|from)\s+selective_state_space_momentum_b200\b", src), f
        assert not re.search(r"CDLL\([^)]*libmmscan|libmmscan\.so\b", src), f
        for inc in re.findall(r'#include\s*[<"]([^>"]+)[>"]', src):
            assert inc in ("math.h", "stddef.h", "stdint.h", "stdlib.h", "string.h"), (f, inc)


def test_missing_library_raises(tmp_path, monkeypatch):
    import selective_state_space_momentum_b200 as mm
    monkeypatch.setattr(mm, "_lib", None)
    monkeypatch.setattr(mm, "_LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="missing"):
        mm.load_library()
    torch = pytest.importorskip("torch")
    x = torch.zeros((1, 4, 16))
    with pytest.raises(RuntimeError, match="missing"):
        mm.mm_scan_fwd(x, x, torch.zeros((4, 16)), x, x, None, None, 0.9, 1.0, x, None, None)
