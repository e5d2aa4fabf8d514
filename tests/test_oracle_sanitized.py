"""The oracle's pins again, with the oracle built under AddressSanitizer and
UndefinedBehaviorSanitizer: an out-of-bounds read or write, a use of freed
memory, a signed overflow or a bad shift anywhere on the pinned paths stops
the run.  The pins run in a child process that preloads the sanitizer
runtimes (the interpreter itself is not instrumented)."""
from __future__ import annotations

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _runtime(name: str) -> str:
    try:
        path = subprocess.run(["gcc", f"-print-file-name={name}"], capture_output=True,
                              text=True, check=True).stdout.strip()
    except (OSError, subprocess.CalledProcessError):
        return ""
    return path if os.path.isabs(path) and os.path.exists(path) else ""


def test_oracle_pins_pass_under_address_and_ub_sanitizers():
    asan, ubsan = _runtime("libasan.so"), _runtime("libubsan.so")
    if not asan or not ubsan:
        pytest.skip("gcc's sanitizer runtimes are not installed")
    env = dict(os.environ, MSA_ORACLE_SANITIZE="1", LD_PRELOAD=f"{asan} {ubsan}",
               ASAN_OPTIONS="detect_leaks=0:halt_on_error=1",
               UBSAN_OPTIONS="print_stacktrace=1:halt_on_error=1", OMP_NUM_THREADS="4")
    tests = ["tests/test_oracle_pins.py", "tests/test_oracle_bwd.py",
             "tests/test_oracle_varlen.py", "tests/test_oracle_project.py",
             "tests/test_oracle_fp8.py"]
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "not gpu",
                        "-p", "no:cacheprovider", *tests],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-3000:])
    assert "passed" in r.stdout
