"""Host thread safety of the library's one-time set-up.

A fresh process (tests/threads_child.py) makes its first library calls from
four host threads at once, each running the whole path on its own stream; all
four results must match the CPU oracle (selection and packing bit-exact,
gradients within the bf16 tolerance).
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_first_calls_from_four_threads():
    r = subprocess.run([sys.executable, "-m", "tests.threads_child"], cwd=ROOT,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "threads ok" in r.stdout
