"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bit-exact: scores, counts, kept, offsets, perm, pos and the packed blocks.
Within tolerance (parity.TOL: 1e-5 fp32, 2e-2 bf16, relative Frobenius per
tensor and per expert): dW_down, dW_gu, dX.  Experts with m_e = 0 must give
exactly zero weight gradients and tokens with no retained pair exactly zero dX.
"""
import numpy as np
import pytest
import torch

from oracle import lrmoe_oracle as O
from pruned_expert_backward_lrmoe_b200 import inputs
from pruned_expert_backward_lrmoe_b200 import lrmoe as L

from tests import parity as PT

pytestmark = pytest.mark.gpu

# Small layers the oracle finishes in seconds; they span several tiles
# (128-row M tiles, 256-column N tiles, 64-deep K blocks) with ragged tails.
SMALL = {
    "tiny": inputs.spec("tiny"),
    "qwen-mini": inputs.spec("qwen", T=512, E=8, k=4, H=256, I=192),
    "ragged": inputs.spec("qwen", T=300, E=6, k=3, H=320, I=136, quota="half_ceil"),
    "skew-mini": inputs.spec("skew", T=1024, E=16, k=4, H=128, I=128),
    "glm-mini": inputs.spec("glm", T=384, E=8, k=8, H=512, I=352, quota="keep:1/4"),
    "f32-ragged": inputs.spec("tiny", T=100, E=5, k=3, H=36, I=20),
    "one-expert": inputs.spec("qwen", T=200, E=1, k=1, H=64, I=64, quota="half_ceil"),
    "full-quota": inputs.spec("qwen", T=256, E=4, k=2, H=128, I=64, quota="full"),
    "over-quota": inputs.spec("qwen", T=256, E=4, k=2, H=128, I=64, quota="over"),
    "zero-quota": inputs.spec("qwen", T=128, E=4, k=2, H=64, I=64, quota="zero"),
    # the limits: E = 1024 experts (grouped-GEMM maximum; the wgrad then uses its
    # 3-stage / 2-buffer layout; most experts empty) and top-32 routing (k maximum)
    "max-sizes": inputs.spec("qwen", T=512, E=1024, k=32, H=64, I=64),
}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    L.load()


@pytest.mark.parametrize("name", list(SMALL))
def test_small_layer_parity(name):
    layer = inputs.make_layer(SMALL[name], seed=0)
    ref = O.pruned_backward(layer)
    out = PT.run_steps(layer)
    M = PT.check_selection(layer, out, ref)
    PT.check_pack(layer, out, ref, M)
    PT.check_gradients(layer, out, ref)
    assert int(out["status"].item()) == 0


@pytest.mark.parametrize("seed", [1, 2])
def test_other_seeds(seed):
    layer = inputs.make_layer(SMALL["qwen-mini"], seed=seed)
    ref = O.pruned_backward(layer)
    out = PT.run_steps(layer)
    M = PT.check_selection(layer, out, ref)
    PT.check_pack(layer, out, ref, M)
    PT.check_gradients(layer, out, ref)


def _same_bytes(a, b):
    return torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8))


def test_chain_entry_point_equals_steps_and_is_deterministic():
    layer = inputs.make_layer(SMALL["ragged"], seed=0)
    inp = PT.device_inputs(layer)
    a = PT.run_steps(layer, inp)
    b = PT.run_chain(layer, inp)
    c = PT.run_chain(layer, inp)
    M = int(a["offsets"][-1].item())
    for name in ("score", "counts", "kept", "offsets", "pos", "dW_down", "dW_gu", "dX"):
        assert _same_bytes(a[name], b[name]), name
        assert _same_bytes(b[name], c[name]), name
    for name in ("perm", "dGUp", "dXp") + PT.chain_packed(layer):
        assert _same_bytes(a[name][:M], b[name][:M]), name
        assert _same_bytes(b[name][:M], c[name][:M]), name


def test_ties_and_duplicates():
    """Many equal scores (identical saved rows) and tokens routed twice to one expert."""
    s = inputs.spec("qwen", T=256, E=4, k=4, H=64, I=64, quota="half_ceil")
    rng = np.random.default_rng(7)
    idx = rng.integers(0, 4, size=(256, 4)).astype(np.int32)   # duplicates allowed
    layer = inputs.make_layer(s, seed=3, topk_idx=idx)
    layer.a[:] = layer.a[0]                                       # every ||a_p|| equal
    layer.dY[:] = layer.dY[0]
    layer.topk_w[:] = np.float32(0.25)                            # every score equal
    ref = O.pruned_backward(layer)
    out = PT.run_steps(layer)
    M = PT.check_selection(layer, out, ref)
    PT.check_pack(layer, out, ref, M)
    PT.check_gradients(layer, out, ref)


def test_invalid_experts_empty_slots_and_nonfinite_scores():
    s = inputs.spec("qwen", T=128, E=4, k=2, H=64, I=64, quota="half_ceil")
    layer = inputs.make_layer(s, seed=4)
    layer.topk_idx[3, 1] = 9      # invalid expert
    layer.topk_idx[5, 0] = -1     # empty slot
    nan_row = O.encode_rne(np.full((1, 64), np.nan, np.float32), "bf16")
    inf_row = O.encode_rne(np.full((1, 64), np.inf, np.float32), "bf16")
    layer.a[7 * 2 + 0] = nan_row[0]
    layer.a[8 * 2 + 1] = inf_row[0]
    score_ref, st_ref = O.lrm_score(layer.topk_idx, layer.topk_w, layer.dY, layer.a, "bf16", 4)
    inp = PT.device_inputs(layer)
    out = L.alloc_buffers(128, 2, 4, 64, 64, torch.bfloat16)
    out["status"].zero_()
    L.lrmoe_score(inp["topk_idx"], inp["topk_w"], inp["dY"], inp["a"], 4, out["score"], out["status"])
    L.lrmoe_select_quota(inp["topk_idx"], out["score"], inp["quota"], out["counts"], out["kept"],
                         out["offsets"], out["perm"], out["pos"], out["workspace"], out["status"])
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out["score"].cpu().numpy().view(np.uint32), score_ref.view(np.uint32))
    counts, kept, offsets, perm, pos, st2 = O.select_quota(layer.topk_idx, score_ref, layer.quota, 4)
    np.testing.assert_array_equal(out["pos"].cpu().numpy(), pos)
    np.testing.assert_array_equal(out["perm"].cpu().numpy()[: perm.size], perm)
    st = int(out["status"].item())
    assert st & L.ST_BAD_EXPERT and st & L.ST_NONFINITE and not st & L.ST_TIMEOUT
    assert st_ref & O.ST_BAD_EXPERT and st_ref & O.ST_NONFINITE


def test_negative_quota_sets_status_and_counts_as_zero():
    s = inputs.spec("qwen", T=128, E=4, k=2, H=64, I=64)
    layer = inputs.make_layer(s, seed=5)
    layer.quota[1] = -3
    ref = O.pruned_backward(layer)
    out = PT.run_steps(layer)
    PT.check_selection(layer, out, ref)
    assert ref["kept"][1] == 0
    assert int(out["status"].item()) & L.ST_BAD_QUOTA
    PT.check_gradients(layer, out, ref)


def test_wgrad_accumulate_adds():
    layer = inputs.make_layer(SMALL["qwen-mini"], seed=0)
    out = PT.run_steps(layer)
    before = out["dW_down"].clone()
    L.lrmoe_grouped_wgrad(out["DYp"], out["Ap"], out["offsets"], out["dW_down"], accumulate=True,
                          status=out["status"])
    torch.cuda.synchronize()
    torch.testing.assert_close(out["dW_down"], 2 * before, rtol=0, atol=0)


# ---------------------------------------------------------------------------
# full-size layers: everything bit-exact that is integer/byte work, gradients
# on sampled experts and tokens
# ---------------------------------------------------------------------------
FULL = ["qwen", "glm", "skew", "sweep100", "sweep25"]


def sampled_experts(kept, rng, n_random=2):
    E = kept.size
    nz = np.nonzero(kept > 0)[0]
    pick = {int(np.argmax(kept))}
    if nz.size:
        pick.add(int(nz[np.argmin(kept[nz])]))
    zero = np.nonzero(kept == 0)[0]
    if zero.size:
        pick.add(int(zero[0]))
    pick.update(int(e) for e in rng.choice(E, size=n_random, replace=False))
    return sorted(pick)


@pytest.mark.slow
@pytest.mark.parametrize("name", FULL)
def test_full_size_parity(name):
    layer = inputs.make_layer(name, seed=0)
    s = layer.spec
    dt = s.dtype
    out = PT.run_chain(layer)
    assert int(out["status"].item()) == 0
    score, _ = O.lrm_score(layer.topk_idx, layer.topk_w, layer.dY, layer.a, dt, s.E)
    counts, kept, offsets, perm, pos, _ = O.select_quota(layer.topk_idx, score, layer.quota, s.E)
    ref = dict(score=score, counts=counts, kept=kept, offsets=offsets, perm=perm, pos=pos)
    M = PT.check_selection(layer, out, ref)
    Xp, DYp, Ap, Gp, Up = O.pack(perm, layer.topk_w, s.k, layer.x, layer.dY, layer.a, layer.g,
                                 layer.u, dt)
    PT.check_pack(layer, out, dict(Xp=Xp, DYp=DYp, Ap=Ap, Gp=Gp, Up=Up), M,
                  PT.chain_packed(layer))
    rng = np.random.default_rng(0)
    experts = sampled_experts(kept, rng)
    dWd, dWgu, _, _ = O.expert_backward(Xp, DYp, Ap, Gp, Up, offsets, layer.W_gu, layer.W_down, dt,
                                        experts=experts)
    tol = PT.TOL[dt]
    got_d = out["dW_down"]
    got_gu = out["dW_gu"]
    for e in experts:
        gd = got_d[e].cpu().numpy()
        gg = got_gu[e].cpu().numpy()
        if kept[e] == 0:
            assert not gd.any() and not gg.any()
            continue
        assert PT.rel_fro(gd, dWd[e]) <= tol, (e, PT.rel_fro(gd, dWd[e]))
        assert PT.rel_fro(gg, dWgu[e]) <= tol, (e, PT.rel_fro(gg, dWgu[e]))
    tokens = sorted(set(rng.choice(s.T, size=48, replace=False).tolist()) | {0, s.T - 1})
    rows = [int(p) for t in tokens for p in pos.reshape(-1, s.k)[t] if p >= 0]
    _, dxp = O.expert_backward_rows(rows, offsets, DYp, Gp, Up, layer.W_gu, layer.W_down, dt)
    want = O.unpack_tokens(tokens, dxp, pos, s.k, s.H)
    got = out["dX"][tokens].float().cpu().numpy()
    assert PT.rel_fro(got, want) <= tol
    # the same bound on every sampled token alone, so that one wrong row cannot
    # hide in the pooled norm
    per_token = [PT.rel_fro(got[i], want[i]) for i in range(len(tokens)) if np.any(want[i])]
    worst = max(per_token) if per_token else 0.0
    print(f"{name}: dX pooled rel err {PT.rel_fro(got, want):.3e}, worst token {worst:.3e}")
    assert worst <= tol, worst
    none = [i for i, t in enumerate(tokens) if (pos.reshape(-1, s.k)[t] < 0).all()]
    assert not got[none].any()
    # invariant that holds at any size: every retained row belongs to its block's expert
    blocks = np.repeat(np.arange(s.E), kept)
    np.testing.assert_array_equal(layer.topk_idx.reshape(-1)[perm], blocks)
