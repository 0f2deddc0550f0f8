"""The library's host planner (lrmoe_redistribute) against the oracle: the same
optimal peak (Hall's condition) and a valid plan, on random copy maps, the
closed forms, and a qwen-sized instance; host-detectable argument errors."""
import time

import numpy as np
import pytest

from oracle import lrmoe_oracle as O
from pruned_expert_backward_lrmoe_b200 import build as B
from pruned_expert_backward_lrmoe_b200 import lrmoe as L


@pytest.fixture(scope="module", autouse=True)
def _lib():
    B.build()


def _valid(plan, m, A, peak):
    assert np.array_equal(plan.sum(axis=1), m)
    assert np.all(plan >= 0) and np.all(plan[~A] == 0)
    assert plan.sum(axis=0).max() == peak or m.sum() == 0


@pytest.mark.parametrize("seed", range(40))
def test_planner_peak_equals_hall_peak(seed):
    rng = np.random.default_rng(seed)
    E, G = int(rng.integers(1, 20)), int(rng.integers(1, 11))
    m = rng.integers(0, 300, size=E) * (rng.random(E) < 0.9)
    A = rng.random((E, G)) < rng.uniform(0.1, 0.7)
    A[np.arange(E), rng.integers(0, G, size=E)] = True
    plan, peak = L.lrmoe_redistribute(m, A)
    assert peak == O.redistribute_peak(m, A)
    _valid(plan, m, A, peak)


def test_planner_closed_forms():
    m = np.array([7, 2, 9, 4, 1])
    assert L.lrmoe_redistribute(m, np.eye(4, dtype=bool)[[0, 1, 1, 3, 2]])[1] == 11
    assert L.lrmoe_redistribute(m, np.ones((5, 3), bool))[1] == 8
    assert L.lrmoe_redistribute(np.zeros(3, np.int64), np.ones((3, 2), bool))[1] == 0


def test_planner_qwen_sized_instance_is_fast():
    """128 experts on 8 GPUs, 16 home experts each plus a second copy of the 16
    hottest (Zipf counts): well under a millisecond per plan on one host core."""
    E, G = 128, 8
    m = (20000 / (np.arange(E) + 1) ** 1.0).astype(np.int64)
    A = np.zeros((E, G), bool)
    A[np.arange(E), np.arange(E) % G] = True
    A[np.arange(16), (np.arange(16) + 3) % G] = True
    t0 = time.perf_counter()
    plan, peak = L.lrmoe_redistribute(m, A)
    dt = time.perf_counter() - t0
    _valid(plan, m, A, peak)
    home = np.zeros(G, np.int64)
    np.add.at(home, np.arange(E) % G, m)
    assert peak <= home.max() and peak >= -(-m.sum() // G)
    assert dt < 0.05


def test_planner_rejects_bad_arguments():
    with pytest.raises(L.LrmoeError):
        L.lrmoe_redistribute([3, 1], np.array([[1, 0], [0, 0]]))   # loaded expert, no copy
    with pytest.raises(L.LrmoeError):
        L.lrmoe_redistribute([-1, 1], np.ones((2, 2)))
    plan, peak = L.lrmoe_redistribute([0, 4], np.array([[0, 0], [1, 1]]))  # empty expert, no copy: fine
    assert peak == 2 and plan[1].sum() == 4
