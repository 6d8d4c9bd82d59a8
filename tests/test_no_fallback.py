"""The product path has no CPU fallback: without libfa_b200.so every entry
point raises, and nothing in the package reaches the oracle (CPU tests)."""

import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "exact_attention_122_b200")


def test_missing_library_raises_on_every_call():
    # A fresh interpreter, so the library handle cached by this process is
    # not reused; the binding is pointed at a path that does not exist.
    code = r"""
import exact_attention_122_b200 as fa
from exact_attention_122_b200 import _binding
_binding.library_path = lambda: "/nonexistent/libfa_b200.so"
_binding._LIB = None
calls = [
    lambda: fa.library(),
    lambda: fa.fa_fwd_raw(0, 0, 0, 0, 0, 1, 1, 1, 64, 0, 1.0, 0),
    lambda: fa.fa_bwd_raw(0, 0, 0, 0, 0, 0, 0, 0, 0, 1, 1, 1, 64, 0, 1.0, 0, 0, 0),
    lambda: fa.fa_fwd_host_raw(0, 0, 0, 0, 0, 1, 1, 1, 64, 0, 1.0, 0, 0, 0),
    lambda: fa.host_workspace_bytes(1, 1, 1, 64),
]
for c in calls:
    try:
        c()
    except ImportError as e:
        assert "missing" in str(e)
    else:
        raise SystemExit("an entry point ran without the library")
print("all raised")
"""
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "all raised" in r.stdout


def test_package_never_imports_the_oracle():
    """No module of the package imports the oracle; the runtime modules (the
    binding, autograd, build) do not even import numpy.  csrc/ holds only the
    CUDA sources."""
    oracle_pat = re.compile(r"^\s*(import\s+oracle|from\s+oracle\b)", re.M)
    numpy_pat = re.compile(r"^\s*(import\s+numpy|from\s+numpy\b)", re.M)
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith(".py"):
                path = os.path.join(dirpath, f)
                text = open(path).read()
                assert not oracle_pat.search(text), path
                if dirpath == PKG:
                    assert not numpy_pat.search(text), path
