"""The SwiGLU epilogue that reads g, u in place (row perm[r]) instead of packed
G_p, U_p: bit-identical to the packed variant; out-of-range perm entries are
flagged and their rows skipped; pack leaves G_p, U_p alone when not asked."""
import numpy as np
import pytest
import torch

from pruned_expert_backward_lrmoe_b200 import inputs
from pruned_expert_backward_lrmoe_b200 import lrmoe as L
from tests import parity as PT

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,over", [("qwen", dict(T=600, E=16, H=256, I=192)),
                                       ("glm", dict(T=300, E=8, H=512, I=320)),
                                       ("skew", dict(T=700, E=16, H=256, I=136))])
def test_gather_equals_packed(name, over):
    layer = inputs.make_layer(inputs.spec(name, **over), seed=16)
    s = layer.spec
    inp = PT.device_inputs(layer)
    out = PT.run_steps(layer, inp)
    M = int(out["offsets"][-1].item())
    got = torch.full_like(out["dGUp"], float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.lrmoe_grouped_dgrad_swiglu_gather(out["DYp"], inp["W_down"], out["offsets"], out["perm"],
                                        inp["g"], inp["u"], got, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(got[:M].view(torch.int16), out["dGUp"][:M].view(torch.int16))


def test_gather_flags_bad_perm_entries():
    layer = inputs.make_layer(inputs.spec("qwen", T=200, E=8, H=128, I=64), seed=17)
    s = layer.spec
    inp = PT.device_inputs(layer)
    out = PT.run_steps(layer, inp)
    perm = out["perm"].clone()
    perm[0] = s.P + 5                  # past the end of g, u
    got = torch.full_like(out["dGUp"], float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.lrmoe_grouped_dgrad_swiglu_gather(out["DYp"], inp["W_down"], out["offsets"], perm,
                                        inp["g"], inp["u"], got, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & L.ST_BAD_INDEX
    M = int(out["offsets"][-1].item())
    assert torch.isnan(got[0].float()).all()                     # skipped row left alone
    assert torch.equal(got[1:M].view(torch.int16), out["dGUp"][1:M].view(torch.int16))


def test_pack_without_g_u_leaves_them_alone():
    layer = inputs.make_layer(inputs.spec("qwen", T=200, E=8, H=128, I=64), seed=18)
    inp = PT.device_inputs(layer)
    out = PT.run_steps(layer, inp)
    bufs = {n: torch.full_like(out[n], float("nan")) for n in ("Xp", "DYp", "Ap")}
    L.lrmoe_pack(out["perm"], out["offsets"], inp["topk_w"], inp["x"], inp["dY"], inp["a"], None,
                 None, bufs["Xp"], bufs["DYp"], bufs["Ap"], None, None, out["status"])
    torch.cuda.synchronize()
    M = int(out["offsets"][-1].item())
    for n in bufs:
        assert torch.equal(bufs[n][:M].view(torch.int16), out[n][:M].view(torch.int16)), n


@pytest.mark.parametrize("name,over", [("qwen", dict(T=600, E=16, H=256, I=192)),
                                       ("glm", dict(T=300, E=8, H=512, I=320)),
                                       ("skew", dict(T=700, E=16, H=256, I=136)),
                                       ("qwen", dict(T=64, E=32, H=128, I=64))])
@pytest.mark.parametrize("accumulate", [False, True])
def test_wgrad_gather_equals_packed(name, over, accumulate):
    """dW_down from a[perm] and dW_gu from x[perm / k] equal the wgrads on packed rows."""
    layer = inputs.make_layer(inputs.spec(name, **over), seed=19)
    s = layer.spec
    inp = PT.device_inputs(layer)
    out = PT.run_steps(layer, inp)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    for grad, src, div, packed, dw in (("DYp", inp["a"], 1, "Ap", "dW_down"),
                                       ("dGUp", inp["x"], s.k, "Xp", "dW_gu")):
        base = torch.randn_like(out[dw]) if accumulate else None
        want = base.clone() if accumulate else torch.full_like(out[dw], float("nan"))
        got = base.clone() if accumulate else torch.full_like(out[dw], float("nan"))
        L.lrmoe_grouped_wgrad(out[grad], out[packed], out["offsets"], want, accumulate=accumulate,
                              status=st)
        L.lrmoe_grouped_wgrad_gather(out[grad], out["perm"], src, div, s.P, out["offsets"], got,
                                     accumulate=accumulate, status=st)
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int32), want.view(torch.int32)), dw
    assert int(st.item()) == 0


def test_wgrad_gather_flags_bad_perm_entries():
    layer = inputs.make_layer(inputs.spec("qwen", T=200, E=8, H=128, I=64), seed=20)
    s = layer.spec
    inp = PT.device_inputs(layer)
    out = PT.run_steps(layer, inp)
    perm = out["perm"].clone()
    perm[1] = -3
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dw = torch.empty_like(out["dW_down"])
    L.lrmoe_grouped_wgrad_gather(out["DYp"], perm, inp["a"], 1, s.P, out["offsets"], dw, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & L.ST_BAD_INDEX
    assert torch.isfinite(dw).all()


def test_pack_dy_only():
    layer = inputs.make_layer(inputs.spec("qwen", T=200, E=8, H=128, I=64), seed=21)
    inp = PT.device_inputs(layer)
    out = PT.run_steps(layer, inp)
    dyp = torch.full_like(out["DYp"], float("nan"))
    L.lrmoe_pack(out["perm"], out["offsets"], inp["topk_w"], None, inp["dY"], None, None, None,
                 None, dyp, None, None, None, out["status"])
    torch.cuda.synchronize()
    M = int(out["offsets"][-1].item())
    assert torch.equal(dyp[:M].view(torch.int16), out["DYp"][:M].view(torch.int16))
