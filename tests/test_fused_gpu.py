"""lrmoe_grouped_dgrad_wgrad (one launch for a dgrad and a wgrad over the same
gradient rows) equals the two separate calls bit for bit, for both epilogues,
ragged and empty experts, and accumulation; and the oracle within tolerance."""
import numpy as np
import pytest
import torch

from oracle import lrmoe_oracle as O
from pruned_expert_backward_lrmoe_b200 import inputs
from pruned_expert_backward_lrmoe_b200 import lrmoe as L
from tests import parity as PT

pytestmark = pytest.mark.gpu

CASES = [("qwen", dict(T=600, E=16, H=256, I=192)),
         ("glm", dict(T=300, E=8, H=512, I=320)),
         ("skew", dict(T=700, E=16, H=256, I=128)),
         ("qwen", dict(T=64, E=32, H=128, I=64))]          # many empty experts


def _pairs(out, inp):
    """(grad rows, W, epilogue, dgrad out, wgrad in rows, dW) of the two GEMM pairs."""
    return [("DYp", inp["W_down"], L.LRMOE_EPI_SWIGLU_BWD, "dGUp", "Ap", "dW_down"),
            ("dGUp", inp["W_gu"], L.LRMOE_EPI_STORE, "dXp", "Xp", "dW_gu")]


@pytest.mark.parametrize("name,over", CASES)
@pytest.mark.parametrize("accumulate", [False, True])
def test_fused_equals_separate_calls(name, over, accumulate):
    layer = inputs.make_layer(inputs.spec(name, **over), seed=14)
    inp = PT.device_inputs(layer)
    out = PT.run_steps(layer, inp)
    st = out["status"]
    for grad, W, epi, dout, inrows, dw in _pairs(out, inp):
        kw = dict(Gp=out["Gp"], Up=out["Up"]) if epi == L.LRMOE_EPI_SWIGLU_BWD else {}
        base = torch.randn_like(out[dw]) if accumulate else None
        sep_out, fus_out = torch.full_like(out[dout], float("nan")), torch.full_like(out[dout], float("nan"))
        sep_dw = base.clone() if accumulate else torch.full_like(out[dw], float("nan"))
        fus_dw = base.clone() if accumulate else torch.full_like(out[dw], float("nan"))
        L.lrmoe_grouped_dgrad(out[grad], W, out["offsets"], epi, sep_out, status=st, **kw)
        L.lrmoe_grouped_wgrad(out[grad], out[inrows], out["offsets"], sep_dw,
                              accumulate=accumulate, status=st)
        L.lrmoe_grouped_dgrad_wgrad(out[grad], W, out["offsets"], epi, fus_out, out[inrows],
                                    fus_dw, accumulate=accumulate, status=st, **kw)
        torch.cuda.synchronize()
        M = int(out["offsets"][-1].item())
        assert torch.equal(sep_out[:M].view(torch.int16), fus_out[:M].view(torch.int16))
        assert torch.equal(sep_dw.view(torch.int32), fus_dw.view(torch.int32))
    assert int(st.item()) == 0


def test_fused_path_matches_oracle():
    """The path with both GEMM pairs fused (each after a NaN fill of its outputs)."""
    layer = inputs.make_layer(inputs.spec("qwen", T=512, E=16, H=256, I=192), seed=15)
    s = layer.spec
    inp = PT.device_inputs(layer)
    out = PT.run_steps(layer, inp)
    st = out["status"]
    for name in ("dGUp", "dW_down", "dXp", "dW_gu", "dX"):
        out[name].fill_(float("nan"))
    L.lrmoe_grouped_dgrad_wgrad(out["DYp"], inp["W_down"], out["offsets"], L.LRMOE_EPI_SWIGLU_BWD,
                                out["dGUp"], out["Ap"], out["dW_down"], Gp=out["Gp"],
                                Up=out["Up"], status=st)
    L.lrmoe_grouped_dgrad_wgrad(out["dGUp"], inp["W_gu"], out["offsets"], L.LRMOE_EPI_STORE,
                                out["dXp"], out["Xp"], out["dW_gu"], status=st)
    L.lrmoe_unpack(out["dXp"], out["pos"], s.T, s.k, out["dX"], st)
    torch.cuda.synchronize()
    ref = O.pruned_backward(layer)
    PT.check_selection(layer, out, ref)
    PT.check_gradients(layer, out, ref)
    assert int(st.item()) == 0


def test_fused_rejects_fp32():
    layer = inputs.make_layer(inputs.spec("tiny", T=64), seed=1)
    inp = PT.device_inputs(layer)
    out = PT.run_steps(layer, inp)
    with pytest.raises(L.LrmoeError) as ei:
        L.lrmoe_grouped_dgrad_wgrad(out["DYp"], inp["W_down"], out["offsets"],
                                    L.LRMOE_EPI_SWIGLU_BWD, out["dGUp"], out["Ap"],
                                    out["dW_down"], Gp=out["Gp"], Up=out["Up"])
    assert ei.value.code == L.LRMOE_ERR_UNSUPPORTED
