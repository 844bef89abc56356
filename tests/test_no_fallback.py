"""The product path has no CPU fallback and never touches the oracle (CPU only).

The binding loads libs2attn.so and nothing else: without the library every
call raises, and importing the package (binding, sequence-parallel layer,
synthetic inputs) loads no module of the oracle.
"""
from __future__ import annotations

import subprocess
import sys
from pathlib import Path

import pytest
import torch

ROOT = Path(__file__).resolve().parent.parent


def test_missing_library_raises(monkeypatch, tmp_path):
    from shifted_sparse_attention_b200 import binding as s2

    monkeypatch.setattr(s2, "LIB_PATH", tmp_path / "libs2attn.so")
    monkeypatch.setattr(s2, "_lib", None)
    with pytest.raises(ImportError):
        s2.lib()
    x = torch.zeros(1, 256, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(Exception):
        s2.forward(x, x, x, 256)


def test_package_imports_no_oracle_module():
    code = ("import sys; import shifted_sparse_attention_b200.binding, shifted_sparse_attention_b200.sp, "
            "shifted_sparse_attention_b200.synthetic; "
            "bad = [m for m in sys.modules if m == 'oracle' or m.startswith('oracle.')]; "
            "print(bad); sys.exit(1 if bad else 0)")
    r = subprocess.run([sys.executable, "-c", code], cwd=str(ROOT), capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr[-2000:]
