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


def test_send_slots_of_the_packed_rows():
    """row_dest from the split equals the oracle's send positions, bit for bit."""
    layer = inputs.make_layer(inputs.spec("qwen", T=600, E=16, H=64, I=64), seed=14)
    s = layer.spec
    out = PT.run_steps(layer)
    kept = out["kept"].cpu().numpy().astype(np.int64)
    start = np.arange(s.E) % 3                     # as if lower ranks held a few rows
    plan, _ = L.lrmoe_redistribute(kept + start, _copy_map(s.E, 4, 7))
    rd = torch.full((s.P,), -7, dtype=torch.int32, device="cuda")
    pd = torch.full((s.P,), -7, dtype=torch.int32, device="cuda")
    do = torch.full((5,), -7, dtype=torch.int32, device="cuda")
    deo = torch.full((4, s.E + 1), -7, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.lrmoe_split_by_destination(out["perm"], out["offsets"],
                                 torch.from_numpy(plan.astype(np.int32)).cuda(), pd, do, deo,
                                 global_start=torch.from_numpy(start.astype(np.int32)).cuda(),
                                 status=st, row_dest=rd)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    M = int(kept.sum())
    want = O.send_positions(out["perm"].cpu().numpy(), pd.cpu().numpy(), M)
    np.testing.assert_array_equal(rd.cpu().numpy()[:M], want)
    assert (rd.cpu().numpy()[M:] == -7).all()


@pytest.mark.parametrize("G,E,seed", [(1, 8, 0), (3, 16, 1), (8, 128, 2), (5, 1024, 3)])
def test_group_received_matches_the_oracle(G, E, seed):
    rng = np.random.default_rng(seed)
    cnt = rng.integers(0, 5, size=(G, E)) * (rng.random((G, E)) < 0.6)
    tab = np.concatenate([np.zeros((G, 1), np.int64), np.cumsum(cnt, axis=1)], axis=1)
    R = int(tab[:, E].sum())
    cap = R + 3
    order = torch.full((cap,), -7, dtype=torch.int32, device="cuda")
    inv = torch.full((cap,), -7, dtype=torch.int32, device="cuda")
    offs = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.lrmoe_group_received(torch.from_numpy(tab.astype(np.int32)).cuda(), order, inv, offs, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    o, i, off = O.group_received(tab)
    np.testing.assert_array_equal(order.cpu().numpy()[:R], o)
    np.testing.assert_array_equal(inv.cpu().numpy()[:R], i)
    np.testing.assert_array_equal(offs.cpu().numpy(), off)
    assert (order.cpu().numpy()[R:] == -7).all()


def test_group_received_flags_a_table_larger_than_its_buffers():
    tab = torch.tensor([[0, 3, 5], [0, 2, 2]], dtype=torch.int32, device="cuda")   # 7 rows
    order = torch.full((4,), -7, dtype=torch.int32, device="cuda")
    inv = torch.full((4,), -7, dtype=torch.int32, device="cuda")
    offs = torch.empty(3, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.lrmoe_group_received(tab, order, inv, offs, st)
    torch.cuda.synchronize()
    assert int(st.item()) & L.ST_BAD_INDEX
    assert offs.cpu().tolist() == [0, 5, 7]


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_exchange_rows_pack_and_split(dt):
    """lrmoe_pack_wide writes [x | w dY | a | g | u] = the oracle's packed rows side by
    side; lrmoe_split_wide takes rows by an index list back into the five blocks."""
    over = dict(T=500, E=8, H=128, I=64) if dt == "bf16" else dict(T=300, E=8, H=36, I=20)
    layer = inputs.make_layer(inputs.spec("qwen" if dt == "bf16" else "tiny", **over), seed=15)
    s = layer.spec
    inp = PT.device_inputs(layer)
    out = PT.run_steps(layer, inp)
    kept = out["kept"].cpu().numpy().astype(np.int64)
    plan, _ = L.lrmoe_redistribute(kept, _copy_map(s.E, 3, 4))
    pd, do, deo, st = _split(out, plan, s.E, 3)
    W = 2 * s.H + 3 * s.I
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    rows = torch.full((s.P, W), float("nan"), dtype=tdt, device="cuda")
    L.lrmoe_pack_wide(pd, do, inp["topk_w"], inp["x"], inp["dY"], inp["a"], inp["g"], inp["u"],
                      rows, out["status"])
    torch.cuda.synchronize()
    M = int(do[-1].item())
    ref = O.pack(pd.cpu().numpy()[:M], layer.topk_w, s.k, layer.x, layer.dY, layer.a, layer.g,
                 layer.u, s.dtype)
    want = np.concatenate([np.asarray(r) for r in ref], axis=1)
    np.testing.assert_array_equal(PT.to_numpy_storage(rows[:M], s.dtype), want)
    idx_np = np.random.default_rng(1).permutation(M).astype(np.int32)
    idx = torch.from_numpy(idx_np).cuda()
    parts = {n: torch.empty(M, s.H if n in ("Xp", "DYp") else s.I, dtype=tdt, device="cuda")
             for n in ("Xp", "DYp", "Ap", "Gp", "Up")}
    L.lrmoe_split_wide(rows, idx, parts["Xp"], parts["DYp"], parts["Ap"], parts["Gp"], parts["Up"],
                       out["status"])
    torch.cuda.synchronize()
    assert int(out["status"].item()) == 0
    for n, r in zip(("Xp", "DYp", "Ap", "Gp", "Up"), ref):
        np.testing.assert_array_equal(PT.to_numpy_storage(parts[n], s.dtype), np.asarray(r)[idx_np])
