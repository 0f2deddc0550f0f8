"""Split of the packed rows by destination on the GPU against the oracle, bit for
bit (one rank, and a second rank's rows through global_start), the coverage
check, and the send buffer gathered by lrmoe_pack from perm_dest."""
import numpy as np
import pytest
import torch

from oracle import lrmoe_oracle as O
from pruned_expert_backward_lrmoe_b200 import inputs
from pruned_expert_backward_lrmoe_b200 import lrmoe as L
from tests import parity as PT

pytestmark = pytest.mark.gpu


def _copy_map(E, G, seed):
    rng = np.random.default_rng(seed)
    A = rng.random((E, G)) < 0.35
    A[np.arange(E), np.arange(E) % G] = True
    return A


def _split(out, plan, E, G, start=None):
    rows_cap = out["perm"].shape[0]
    pd = torch.full((rows_cap,), -7, dtype=torch.int32, device="cuda")
    do = torch.full((G + 1,), -7, dtype=torch.int32, device="cuda")
    deo = torch.full((G, E + 1), -7, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.lrmoe_split_by_destination(out["perm"], out["offsets"],
                                 torch.from_numpy(plan.astype(np.int32)).cuda(), pd, do, deo,
                                 global_start=None if start is None else
                                 torch.from_numpy(np.asarray(start, np.int32)).cuda(), status=st)
    torch.cuda.synchronize()
    return pd, do, deo, int(st.item())


def _check(out, plan, pd, do, deo, start=None):
    perm = out["perm"].cpu().numpy()
    offsets = out["offsets"].cpu().numpy()
    rpd, rdo, rdeo = O.split_by_destination(perm, offsets, plan, start)
    np.testing.assert_array_equal(do.cpu().numpy(), rdo)
    np.testing.assert_array_equal(deo.cpu().numpy(), rdeo)
    np.testing.assert_array_equal(pd.cpu().numpy()[: rdo[-1]], rpd)


@pytest.mark.parametrize("G", [1, 3, 8])
def test_split_one_rank(G):
    layer = inputs.make_layer(inputs.spec("qwen", T=700, E=16, H=64, I=64), seed=11)
    s = layer.spec
    out = PT.run_steps(layer)
    kept = out["kept"].cpu().numpy().astype(np.int64)
    plan, peak = L.lrmoe_redistribute(kept, _copy_map(s.E, G, G))
    pd, do, deo, st = _split(out, plan, s.E, G)
    assert st == 0
    _check(out, plan, pd, do, deo)
    assert int(do[-1].item()) == int(kept.sum())


def test_split_two_ranks_share_one_plan():
    """Rank 0 and rank 1 hold different tokens of the same layer; the plan is made
    from their summed counts; each rank's split follows its global offset."""
    spec = inputs.spec("qwen", T=400, E=8, H=64, I=64)
    outs = [PT.run_steps(inputs.make_layer(spec, seed=20 + r)) for r in range(2)]
    kept = [o["kept"].cpu().numpy().astype(np.int64) for o in outs]
    plan, _ = L.lrmoe_redistribute(kept[0] + kept[1], _copy_map(spec.E, 4, 5))
    served = np.zeros_like(plan)
    for r, start in enumerate([np.zeros(spec.E, np.int64), kept[0]]):
        pd, do, deo, st = _split(outs[r], plan, spec.E, 4, start)
        assert st == 0
        _check(outs[r], plan, pd, do, deo, start)
        served += np.diff(deo.cpu().numpy(), axis=1).T
    np.testing.assert_array_equal(served, plan)


def test_split_flags_rows_the_plan_does_not_cover():
    layer = inputs.make_layer(inputs.spec("qwen", T=300, E=8, H=64, I=64), seed=12)
    out = PT.run_steps(layer)
    kept = out["kept"].cpu().numpy().astype(np.int64)
    plan, _ = L.lrmoe_redistribute(kept, np.ones((8, 2), bool))
    e = int(np.argmax(kept))
    plan[e, int(np.argmax(plan[e]))] -= 1    # one row of expert e has no destination
    pd, do, deo, st = _split(out, plan, 8, 2)
    assert st & L.ST_BAD_INDEX
    assert int(do[-1].item()) == int(kept.sum()) - 1


def test_send_buffer_packed_from_perm_dest():
    layer = inputs.make_layer(inputs.spec("qwen", T=500, E=8, H=128, I=64), seed=13)
    s = layer.spec
    inp = PT.device_inputs(layer)
    out = PT.run_steps(layer, inp)
    kept = out["kept"].cpu().numpy().astype(np.int64)
    plan, _ = L.lrmoe_redistribute(kept, _copy_map(s.E, 4, 3))
    pd, do, deo, st = _split(out, plan, s.E, 4)
    bufs = {n: torch.empty_like(out[n]) for n in ("Xp", "DYp", "Ap", "Gp", "Up")}
    L.lrmoe_pack(pd, do, inp["topk_w"], inp["x"], inp["dY"], inp["a"], inp["g"], inp["u"],
                 bufs["Xp"], bufs["DYp"], bufs["Ap"], bufs["Gp"], bufs["Up"], out["status"])
    torch.cuda.synchronize()
    M = int(do[-1].item())
    ref = O.pack(pd.cpu().numpy()[:M], layer.topk_w, s.k, layer.x, layer.dY, layer.a, layer.g,
                 layer.u, s.dtype)
    for name, r in zip(("Xp", "DYp", "Ap", "Gp", "Up"), ref):
        got = PT.to_numpy_storage(bufs[name][:M], s.dtype)
        np.testing.assert_array_equal(got, r)
