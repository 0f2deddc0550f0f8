"""Quota controller on the GPU against the oracle (integer outputs: bit-exact),
including the configs' capacity rule, budgets that cut, and edge cases."""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import lrmoe_oracle as O
from pruned_expert_backward_lrmoe_b200 import inputs
from pruned_expert_backward_lrmoe_b200 import lrmoe as L

pytestmark = pytest.mark.gpu


def _run(idx, E, cap, budget):
    t = torch.from_numpy(np.ascontiguousarray(idx, np.int32)).cuda()
    q = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    c = torch.full((E,), -7, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.lrmoe_quota_controller(t, E, cap, budget, q, c, st)
    torch.cuda.synchronize()
    return q.cpu().numpy(), c.cpu().numpy(), int(st.item())


@pytest.mark.parametrize("name", ["qwen", "skew"])
@pytest.mark.parametrize("frac", [None, 1.0, 0.3, 0.05, 0.0])
def test_controller_matches_oracle(name, frac):
    layer = inputs.make_layer(inputs.spec(name, T=2048, E=64, H=64, I=64), seed=1)
    s = layer.spec
    P = s.P
    cap = (s.T * s.k) // s.E if frac is None else 0
    budget = -1 if frac is None else int(frac * P)
    q, c, st = _run(layer.topk_idx, s.E, cap, budget)
    q_ref, c_ref = O.quota_controller(layer.topk_idx, s.E, cap, budget)
    np.testing.assert_array_equal(c, c_ref)
    np.testing.assert_array_equal(q, q_ref)
    assert st == 0
    if frac is None:  # cap = T*k/E and no budget is the configs' "capacity" quota rule
        np.testing.assert_array_equal(
            q, inputs.quota_from_counts(layer.counts, dataclasses.replace(s, quota="capacity")))


def test_controller_ragged_and_invalid_ids():
    rng = np.random.default_rng(3)
    idx = rng.integers(-1, 12, size=(1001, 3)).astype(np.int32)   # P not a multiple of 4
    q, c, st = _run(idx, 10, 50, 700)
    q_ref, c_ref = O.quota_controller(idx, 10, 50, 700)
    np.testing.assert_array_equal(c, c_ref)
    np.testing.assert_array_equal(q, q_ref)
    assert st & L.ST_BAD_EXPERT


def test_controller_feeds_selection_on_device():
    """Controller -> select on one stream equals the oracle chain with the same quotas."""
    layer = inputs.make_layer(inputs.spec("qwen", T=1024, E=16, H=64, I=64), seed=2)
    s = layer.spec
    budget = s.P // 5
    q_ref, _ = O.quota_controller(layer.topk_idx, s.E, 0, budget)
    from tests import parity as PT
    inp = PT.device_inputs(layer)
    out = L.alloc_buffers(s.T, s.k, s.E, s.H, s.I, torch.bfloat16)
    st = out["status"]
    st.zero_()
    counts = torch.empty(s.E, dtype=torch.int32, device="cuda")
    L.lrmoe_quota_controller(inp["topk_idx"], s.E, 0, budget, inp["quota"], counts, st)
    L.lrmoe_pruned_backward(inp, out)
    torch.cuda.synchronize()
    layer.quota = q_ref
    ref = O.pruned_backward(layer)
    PT.check_selection(layer, out, ref)
    PT.check_gradients(layer, out, ref)
    assert int(out["offsets"][-1].item()) <= budget
