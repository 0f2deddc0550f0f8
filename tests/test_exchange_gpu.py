"""The redistributed backward module on one GPU (world size 1: one destination,
so the split, the exchange and the regrouping are identities) equals the chain
entry point bit for bit; and the row gather it uses."""
import numpy as np
import pytest
import torch

from pruned_expert_backward_lrmoe_b200 import exchange as X
from pruned_expert_backward_lrmoe_b200 import inputs
from pruned_expert_backward_lrmoe_b200 import lrmoe as L
from tests import parity as PT

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,over", [("qwen", dict(T=512, E=16, H=256, I=192)),
                                       ("skew", dict(T=700, E=16, H=128, I=136))])
def test_world_one_equals_chain(name, over):
    layer = inputs.make_layer(inputs.spec(name, **over), seed=24)
    s = layer.spec
    inp = PT.device_inputs(layer)
    ref = PT.run_chain(layer, inp)
    stats = {}
    got = X.redistributed_backward(inp, np.ones((s.E, 1), bool), stats=stats)
    torch.cuda.synchronize()
    assert int(got["status"].item()) == 0
    for n in ("dW_down", "dW_gu", "dX"):
        assert torch.equal(got[n].view(torch.uint8), ref[n].view(torch.uint8)), n
    assert stats["peak"] == int(ref["offsets"][-1].item())


def test_gather_rows():
    src = torch.randn(100, 48, device="cuda").to(torch.bfloat16)      # 96-byte rows
    idx = torch.tensor([5, 0, 99, 5, 42], dtype=torch.int32, device="cuda")
    dst = torch.full((5, 48), float("nan"), device="cuda").to(torch.bfloat16)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.lrmoe_gather_rows(src, idx, dst, st)
    torch.cuda.synchronize()
    assert torch.equal(dst.view(torch.int16), src[idx.long()].view(torch.int16))
    bad = torch.tensor([1, 100], dtype=torch.int32, device="cuda")
    dst2 = torch.zeros(2, 48, device="cuda").to(torch.bfloat16)
    L.lrmoe_gather_rows(src, bad, dst2, st)
    torch.cuda.synchronize()
    assert int(st.item()) & L.ST_BAD_INDEX
    assert torch.equal(dst2[0].view(torch.int16), src[1].view(torch.int16))
    assert torch.count_nonzero(dst2[1].float()) == 0                 # left unwritten
