"""Failure detection on the GPU without a fault: a bounded device wait on a
barrier that nothing completes must give up, report LRMOE_ST_TIMEOUT in the
status word and leave the context usable for the next call."""
import time

import pytest
import torch

from pruned_expert_backward_lrmoe_b200 import inputs
from pruned_expert_backward_lrmoe_b200 import lrmoe as L

from tests import parity as PT

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    L.lrmoe_selftest_bounded_wait(2000, status)     # 2 ms limit
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    st = int(status.item())
    assert st & L.ST_TIMEOUT
    assert not st & L.ST_BAD_INDEX                   # the wait never "succeeded"
    assert elapsed < 1.0
    # the context still runs the real path correctly afterwards
    layer = inputs.make_layer(inputs.spec("qwen", T=128, E=4, k=2, H=64, I=64), seed=0)
    out = PT.run_chain(layer)
    assert int(out["status"].item()) == 0
    from oracle import lrmoe_oracle as O
    ref = O.pruned_backward(layer)
    PT.check_selection(layer, out, ref)
    PT.check_gradients(layer, out, ref)
