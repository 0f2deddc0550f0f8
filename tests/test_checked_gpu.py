"""The checked-index debug build (liblrmoe_checked.so, compiled with
-DLRMOE_CHECKED): same results as the normal build on valid inputs, and a
status bit instead of stray memory accesses when a grouped GEMM's offsets break
their contract.  Runs in child processes (the binding picks its library once per
process), with the two-SM and the one-SM grouped-GEMM tiles."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "pruned_expert_backward_lrmoe_b200", "liblrmoe_checked.so")


@pytest.mark.parametrize("one_sm", [False, True])
def test_checked_build(one_sm):
    assert os.path.exists(LIB), "build it with `python -m pruned_expert_backward_lrmoe_b200.build --checked`"
    env = dict(os.environ, LRMOE_CHECKED="1")
    env.pop("LRMOE_GEMM_ONE_SM", None)
    if one_sm:
        env["LRMOE_GEMM_ONE_SM"] = "1"
    r = subprocess.run([sys.executable, "-m", "tests.checked_child"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "checked ok" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]
