"""The product path has no fallback: without libsla.so every call raises, and
importing the package loads nothing from the oracle (CPU only)."""
import os
import subprocess
import sys

import pytest

import block_sparse_linear_proj_b200 as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_calls_raise_without_the_library(monkeypatch, tmp_path):
    monkeypatch.setattr(S.sla, "LIB_PATH", str(tmp_path / "libsla.so"))
    monkeypatch.setattr(S.sla, "_lib", None)
    with pytest.raises(ImportError):
        S.sla.load()
    p = S.params(1, 2, 1024, 64, 64, 64, 4)
    with pytest.raises(ImportError):
        S.sla_workspace_size(p)
    with pytest.raises(ImportError):
        S.workspace(p)


def test_package_import_loads_no_oracle_and_no_library():
    code = ("import sys, block_sparse_linear_proj_b200 as S; "
            "bad = sorted(m for m in sys.modules if m == 'oracle' or m.startswith('oracle.')); "
            "assert not bad, bad; assert S.sla._lib is None; print('ok')")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"
