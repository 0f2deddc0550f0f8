"""The two grouped-GEMM tile shapes give the same bits: the default two-SM tiles
(one tcgen05 MMA per pair of SMs, 256 x 256 output tiles) and the one-SM tiles
(LRMOE_GEMM_ONE_SM=1, 128 x 256 per SM) run the whole path on the same small
layers in two fresh processes; dW_down, dW_gu and dX must be bit-identical."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(path, one_sm):
    env = dict(os.environ)
    env.pop("LRMOE_GEMM_ONE_SM", None)
    if one_sm:
        env["LRMOE_GEMM_ONE_SM"] = "1"
    r = subprocess.run([sys.executable, "-m", "tests.gemm_tiles_child", path], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]


def test_two_sm_and_one_sm_tiles_agree_bit_for_bit(tmp_path):
    a, b = str(tmp_path / "two.npz"), str(tmp_path / "one.npz")
    _run(a, False)
    _run(b, True)
    two, one = np.load(a), np.load(b)
    assert sorted(two.files) == sorted(one.files) and len(two.files) == 15
    for name in two.files:
        assert np.array_equal(two[name].view(np.uint32), one[name].view(np.uint32)), name
