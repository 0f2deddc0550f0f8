"""Routing-weight gradient on the GPU against the oracle, bit for bit: every
routed pair, retained pairs only (pos from the device selection), empty and
invalid slots, ragged pair counts, rows longer than one chunk."""
import numpy as np
import pytest
import torch

from oracle import lrmoe_oracle as O
from pruned_expert_backward_lrmoe_b200 import inputs
from pruned_expert_backward_lrmoe_b200 import lrmoe as L
from tests.parity import storage_tensor

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,over", [("qwen", dict(T=515, E=16, H=2048, I=64)),
                                       ("glm", dict(T=129, E=8, H=4096, I=64)),
                                       ("tiny", dict(T=77)),
                                       ("qwen", dict(T=33, E=8, H=8200, I=64))])
@pytest.mark.parametrize("retained_only", [False, True])
def test_router_grad_bit_exact(name, over, retained_only):
    layer = inputs.make_layer(inputs.spec(name, **over), seed=9)
    s = layer.spec
    idx = layer.topk_idx.copy()
    idx[1, 0] = s.E + 3          # invalid id
    idx[2, s.k - 1] = -1         # empty slot
    y = inputs.saved_expert_outputs(layer)
    pos = None
    if retained_only:
        rng = np.random.default_rng(1)
        pos = np.where(rng.random(s.P) < 0.4, np.arange(s.P), -1).astype(np.int32)
    ref, st_ref = O.router_grad(idx, layer.dY, y, s.dtype, s.E, pos=pos)
    dw = torch.full((s.P,), -7.0, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.lrmoe_router_grad(torch.from_numpy(idx).cuda(), storage_tensor(layer.dY, s.dtype),
                        storage_tensor(y, s.dtype), s.E, dw,
                        pos=None if pos is None else torch.from_numpy(pos).cuda(), status=st)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(dw.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    assert int(st.item()) == st_ref


def test_router_grad_with_device_selection():
    """pos straight from lrmoe_select_quota on the same stream."""
    from tests import parity as PT
    layer = inputs.make_layer(inputs.spec("qwen", T=256, E=8, H=256, I=128), seed=10)
    s = layer.spec
    y = inputs.saved_expert_outputs(layer)
    out = PT.run_chain(layer)
    dw = torch.empty(s.P, device="cuda")
    L.lrmoe_router_grad(torch.from_numpy(layer.topk_idx).cuda(), storage_tensor(layer.dY, s.dtype),
                        storage_tensor(y, s.dtype), s.E, dw, pos=out["pos"])
    torch.cuda.synchronize()
    score, _ = O.lrm_score(layer.topk_idx, layer.topk_w, layer.dY, layer.a, s.dtype, s.E)
    pos = O.select_quota(layer.topk_idx, score, layer.quota, s.E)[4]
    ref, _ = O.router_grad(layer.topk_idx, layer.dY, y, s.dtype, s.E, pos=pos)
    np.testing.assert_array_equal(dw.cpu().numpy().view(np.uint32), ref.view(np.uint32))
