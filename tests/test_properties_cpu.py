"""Property-based checks (hypothesis) of the oracle's selection and of the
library's host planner on small random instances with many ties."""
import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import lrmoe_oracle as O
from pruned_expert_backward_lrmoe_b200 import build as B
from pruned_expert_backward_lrmoe_b200 import lrmoe as L

B.build()


@settings(max_examples=60, deadline=None)
@given(st.data())
def test_selection_is_the_top_quota_by_score_then_pair(data):
    T = data.draw(st.integers(1, 12))
    k = data.draw(st.integers(1, 3))
    E = data.draw(st.integers(1, 4))
    idx = np.array(data.draw(st.lists(st.integers(-1, E), min_size=T * k, max_size=T * k)),
                   np.int32).reshape(T, k)
    # few distinct scores: heavy ties
    score = np.array(data.draw(st.lists(st.sampled_from([0.0, 0.5, 1.0, 2.0]),
                                        min_size=T * k, max_size=T * k)), np.float32)
    quota = np.array(data.draw(st.lists(st.integers(-1, T * k), min_size=E, max_size=E)),
                     np.int32)
    counts, kept, offsets, perm, pos, _ = O.select_quota(idx, score, quota, E)
    flat = idx.reshape(-1)
    for e in range(E):
        pairs = [p for p in range(T * k) if flat[p] == e]
        want = sorted(pairs, key=lambda p: (-float(score[p]), p))[: max(0, min(quota[e], len(pairs)))]
        got = perm[offsets[e]: offsets[e + 1]]
        assert sorted(want) == list(got)
        assert counts[e] == len(pairs) and kept[e] == len(want)
    for p in range(T * k):
        assert (pos[p] >= 0) == (p in set(perm[: offsets[-1]].tolist()))


@settings(max_examples=60, deadline=None)
@given(st.data())
def test_host_planner_reaches_the_hall_peak(data):
    E = data.draw(st.integers(1, 6))
    G = data.draw(st.integers(1, 5))
    m = np.array(data.draw(st.lists(st.integers(0, 40), min_size=E, max_size=E)), np.int64)
    A = np.array(data.draw(st.lists(st.lists(st.booleans(), min_size=G, max_size=G),
                                    min_size=E, max_size=E)), bool)
    A[m > 0] |= ~A[m > 0].any(axis=1, keepdims=True) & (np.arange(G) == 0)  # a copy somewhere
    plan, peak = L.lrmoe_redistribute(m, A)
    assert peak == O.redistribute_peak(m, A)
    assert np.array_equal(plan.sum(axis=1), m) and np.all(plan[~A] == 0) and np.all(plan >= 0)
    if m.sum():
        assert plan.sum(axis=0).max() == peak
