"""Pins of the CPU oracle against things other than itself.

Each test ties one oracle function to a closed form, brute force, a library
routine, finite differences or a hand-worked example, so that a dropped term,
a wrong sign or index, or a transposed operand in the oracle fails here.
No GPU is needed.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import lrmoe_oracle as O
from pruned_expert_backward_lrmoe_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
U = 2.0 ** -24


# ----------------------------------------------------------------------------
# helpers local to the tests
# ----------------------------------------------------------------------------
def brute_force_contribution_norm(w, dy_row, a_row):
    """||(w dY) a^T||_F^2 by forming the full H x I matrix in fp64."""
    G = np.outer(np.float64(w) * dy_row.astype(np.float64), a_row.astype(np.float64))
    return float((G * G).sum())


def small_layer(name="tiny", seed=0, **over):
    return inputs.make_layer(inputs.spec(name, **over), seed=seed)


# ----------------------------------------------------------------------------
# worked example from the golden fixture
# ----------------------------------------------------------------------------
def _read_golden(fname):
    rows = {}
    with open(os.path.join(GOLDEN, fname)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            rows.setdefault(key, []).append([float(v) for v in vals])
    return rows


def test_golden_worked_example():
    g = _read_golden("score_worked_example.txt")
    idx = np.array(g["topk_idx"][0], np.int32).reshape(2, 2)
    w = np.array(g["topk_w"][0], np.float32).reshape(2, 2)
    dY = np.array(g["dY"], np.float32)
    a = np.array(g["a"], np.float32)
    quota = np.array(g["quota"][0], np.int32)
    score, st = O.lrm_score(idx, w, dY, a, "f32", 2)
    assert st == 0
    np.testing.assert_array_equal(score, np.array(g["score"][0], np.float32))
    counts, kept, offsets, perm, pos, st = O.select_quota(idx, score, quota, 2)
    np.testing.assert_array_equal(counts, g["counts"][0])
    np.testing.assert_array_equal(kept, g["kept"][0])
    np.testing.assert_array_equal(offsets, g["offsets"][0])
    np.testing.assert_array_equal(perm, g["perm"][0])
    np.testing.assert_array_equal(pos, g["pos"][0])


# ----------------------------------------------------------------------------
# T1: factorisation of the contribution norm
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_t1_factorisation_dyadic_exact(dtype):
    """Dyadic inputs: brute-force outer-product norm == fp64 factorised == canonical fp32, bitwise."""
    rng = np.random.default_rng(1)
    T, k, E, H, I = 12, 3, 4, 64, 128
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    w = rng.choice(np.array([0.5, 0.25, 0.75, 1.0, 0.125], np.float32), size=(T, k))
    dY32 = (rng.integers(-4, 5, size=(T, H)) / 8.0).astype(np.float32)
    a32 = (rng.integers(-4, 5, size=(T * k, I)) / 8.0).astype(np.float32)
    dY = O.encode_rne(dY32, dtype)
    a = O.encode_rne(a32, dtype)
    s32, st = O.lrm_score(idx, w, dY, a, dtype, E)
    s64 = O.lrm_score_f64(idx, w, dY32, a32)
    for p in range(T * k):
        t = p // k
        bf = brute_force_contribution_norm(w.reshape(-1)[p], dY32[t], a32[p])
        assert bf == s64[p]
        assert float(s32[p]) == bf
    assert st == 0


@pytest.mark.parametrize("dtype,H,I", [("f32", 64, 128), ("bf16", 2048, 768), ("bf16", 4096, 1408),
                                       ("f32", 36, 20)])
def test_t1_factorisation_random_within_bound(dtype, H, I):
    """Random inputs: fp64 factorised vs brute force <= 1e-12, canonical fp32 within its bound."""
    rng = np.random.default_rng(2)
    T, k, E = 16, 2, 3
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    w = rng.random((T, k)).astype(np.float32)
    dY = O.encode_rne(rng.standard_normal((T, H)).astype(np.float32), dtype)
    a = O.encode_rne(rng.standard_normal((T * k, I)).astype(np.float32), dtype)
    dY32, a32 = O.decode(dY, dtype), O.decode(a, dtype)
    s32, _ = O.lrm_score(idx, w, dY, a, dtype, E)
    s64 = O.lrm_score_f64(idx, w, dY32, a32)
    # error of the canonical order: per norm, ceil(D/32) sequential adds + 5 butterfly
    # levels + 1 product rounding; three final multiplies.
    bound = ((math.ceil(H / 32) + 6) + (math.ceil(I / 32) + 6) + 4) * U * 1.01
    for p in range(T * k):
        t = p // k
        if H * I <= 64 * 128:
            bf = brute_force_contribution_norm(w.reshape(-1)[p], dY32[t], a32[p])
            assert abs(bf - s64[p]) <= 1e-12 * bf
        assert abs(float(s32[p]) - s64[p]) <= bound * s64[p]


@pytest.mark.parametrize("dtype,D", [("f32", 64), ("bf16", 64), ("bf16", 776), ("f32", 20)])
def test_row_norm_every_element_counted(dtype, D):
    """A row with one nonzero element at position i has norm x_i^2 exactly, for every i."""
    vals = np.zeros((D, D), np.float32)
    vals[np.arange(D), np.arange(D)] = 1.5 + np.arange(D, dtype=np.float32) / 4
    enc = O.encode_rne(vals, dtype)
    n = O.row_sq_norm(O.decode(enc, dtype), O.VEC[dtype])
    x = O.decode(enc, dtype)[np.arange(D), np.arange(D)].astype(np.float64)
    np.testing.assert_array_equal(n.astype(np.float64), x * x)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_row_norm_lane_partials_then_butterfly(dtype):
    """Hand-worked order check.  Row: 4096 in vector 0 (lane 0) and 1 in vectors 1 and
    3 (lanes 1 and 3).  Lanes 1 and 3 meet at the o=2 step (1 + 1 = 2), which then
    joins 2^24 at o=1: 2^24 + 2 is exact.  A plain left-to-right sum would lose both
    ones (2^24 + 1 rounds to even), giving 2^24."""
    vec = O.VEC[dtype]
    x = np.zeros((1, 32 * vec), np.float32)
    x[0, 0], x[0, vec], x[0, 3 * vec] = 4096.0, 1.0, 1.0
    n = O.row_sq_norm(O.decode(O.encode_rne(x, dtype), dtype), vec)
    assert float(n[0]) == 16777218.0
    seq = np.float32(0.0)
    for v in (4096.0, 1.0, 1.0):                 # the order this pin rules out
        seq = np.float32(seq + np.float32(v * v))
    assert float(seq) == 16777216.0


def test_score_from_saved_norms_equals_score():
    """Splitting the factorisation at ||a_p||^2 changes no bit."""
    layer = small_layer("qwen", seed=3, T=64, E=8, H=64, I=96)
    s = layer.spec
    n_a = O.row_sq_norm(O.decode(layer.a, s.dtype), O.VEC[s.dtype])
    s1, st1 = O.lrm_score(layer.topk_idx, layer.topk_w, layer.dY, layer.a, s.dtype, s.E)
    s2, st2 = O.lrm_score_from_norms(layer.topk_idx, layer.topk_w, layer.dY, n_a, s.dtype, s.E)
    np.testing.assert_array_equal(s1.view(np.uint32), s2.view(np.uint32))
    assert st1 == st2


def test_score_nonrouted_invalid_and_nonfinite():
    T, k, E, H, I = 4, 2, 3, 8, 8
    idx = np.array([[0, -1], [5, 1], [2, 2], [1, 0]], np.int32)
    w = np.full((T, k), 0.5, np.float32)
    dY = np.ones((T, H), np.float32)
    a = np.ones((T * k, I), np.float32)
    a[6, 0] = np.inf            # pair (3,0): score inf
    a[7, 1] = np.nan            # pair (3,1): score NaN
    s, st = O.lrm_score(idx, w, dY, a, "f32", E)
    bits = s.view(np.uint32)
    assert bits[1] == 0 and bits[2] == 0                # not routed / invalid -> +0
    assert st & O.ST_BAD_EXPERT and st & O.ST_NONFINITE
    assert np.isinf(s[6]) and bits[7] == 0x7FFFFFFF
    assert s[0] == 0.25 * 8 * 8


# ----------------------------------------------------------------------------
# bf16 rounding against torch's conversion
# ----------------------------------------------------------------------------
def test_encode_rne_matches_torch():
    rng = np.random.default_rng(3)
    v = rng.standard_normal(200000).astype(np.float32) * np.float32(10.0) ** rng.integers(-40, 39, 200000)
    # exact midpoints (ties) between neighbouring bf16 values, both parities
    base = rng.integers(0, 0x7F00, 20000).astype(np.uint32) << 16
    ties = (base | np.uint32(0x8000)).view(np.float32)
    special = np.array([0.0, -0.0, np.inf, -np.inf, 3.3895313892515355e38, 1e-45, -1e-40,
                        np.float32(3.4028235e38)], np.float32)
    with np.errstate(over="ignore"):
        allv = np.concatenate([v, ties, -ties, special]).astype(np.float32)
    ref = torch.from_numpy(allv).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(O.encode_rne(allv, "bf16"), ref)
    assert O.encode_rne(np.array([np.nan], np.float32), "bf16")[0] == 0x7FFF
    back = O.decode(ref, "bf16")
    np.testing.assert_array_equal(back, torch.from_numpy(allv).to(torch.bfloat16).float().numpy())


# ----------------------------------------------------------------------------
# T3: selection equals a brute-force sort
# ----------------------------------------------------------------------------
def brute_force_select(idx_flat, bits, quota, E):
    P = idx_flat.size
    perm = []
    for e in range(E):
        pairs = [p for p in range(P) if idx_flat[p] == e]
        q = min(max(int(quota[e]), 0), len(pairs))
        ranked = sorted(pairs, key=lambda p: (-int(bits[p]), p))
        perm.extend(sorted(ranked[:q]))
    return perm


SCORE_KINDS = ["random", "ties", "all_equal", "all_zero", "nan_inf"]


@pytest.mark.parametrize("kind", SCORE_KINDS)
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_t3_selection_brute_force(kind, seed):
    rng = np.random.default_rng(100 + seed)
    T, k, E = 97, 3, 7
    idx = rng.integers(-1, E, size=(T, k)).astype(np.int32)
    P = T * k
    if kind == "random":
        s = rng.random(P).astype(np.float32)
    elif kind == "ties":
        s = rng.integers(0, 4, P).astype(np.float32) * np.float32(0.5)
    elif kind == "all_equal":
        s = np.full(P, 1.25, np.float32)
    elif kind == "all_zero":
        s = np.zeros(P, np.float32)
    else:
        s = rng.random(P).astype(np.float32)
        s[rng.integers(0, P, 20)] = np.inf
        s.view(np.uint32)[rng.integers(0, P, 20)] = 0x7FFFFFFF
    quota = rng.integers(-2, 40, size=E).astype(np.int32)
    counts, kept, offsets, perm, pos, st = O.select_quota(idx, s, quota, E)
    ref = brute_force_select(idx.reshape(-1), s.view(np.uint32), quota, E)
    assert perm.tolist() == ref
    assert bool(st & O.ST_BAD_QUOTA) == bool((quota < 0).any())


# ----------------------------------------------------------------------------
# T6 / T7: invariants and nested retained sets
# ----------------------------------------------------------------------------
def check_invariants(idx, score, quota, E, out):
    counts, kept, offsets, perm, pos = out
    flat = idx.reshape(-1)
    bits = score.view(np.uint32)
    for e in range(E):
        c = int(((flat == e)).sum())
        assert counts[e] == c
        assert kept[e] == min(max(int(quota[e]), 0), c)
    assert offsets[0] == 0 and (np.diff(offsets) == kept).all()
    for e in range(E):
        blk = perm[offsets[e]:offsets[e + 1]]
        assert (np.diff(blk) > 0).all()
        assert (flat[blk] == e).all()
        dropped = np.setdiff1d(np.nonzero(flat == e)[0], blk)
        if blk.size and dropped.size:
            assert bits[blk].min() >= bits[dropped].max()
    assert (pos[perm] == np.arange(perm.size)).all()
    mask = np.ones(flat.size, bool)
    mask[perm] = False
    assert (pos[mask] == -1).all()


@pytest.mark.parametrize("name,over", [("tiny", {}), ("qwen", dict(T=256, E=16, H=64, I=64)),
                                       ("skew", dict(T=512, E=32, H=64, I=64))])
def test_t6_invariants(name, over):
    L = small_layer(name, **over)
    s, _ = O.lrm_score(L.topk_idx, L.topk_w, L.dY, L.a, L.dtype, L.spec.E)
    out = O.select_quota(L.topk_idx, s, L.quota, L.spec.E)
    check_invariants(L.topk_idx, s, L.quota, L.spec.E, out[:5])
    r = O.pruned_backward(L)
    for e in range(L.spec.E):
        if r["kept"][e] == 0:
            assert not r["dW_down"][e].any() and not r["dW_gu"][e].any()
    pos = r["pos"].reshape(L.spec.T, L.spec.k)
    none_kept = (pos < 0).all(axis=1)
    assert not r["dX"][none_kept].any()


def test_t7_monotone_quota():
    L = small_layer("tiny")
    E = L.spec.E
    s, _ = O.lrm_score(L.topk_idx, L.topk_w, L.dY, L.a, L.dtype, E)
    prev = set()
    for q in range(0, int(L.counts.max()) + 2, 3):
        quota = np.full(E, q, np.int32)
        perm = O.select_quota(L.topk_idx, s, quota, E)[3]
        cur = set(perm.tolist())
        assert prev <= cur
        prev = cur


# ----------------------------------------------------------------------------
# T2: full quota reproduces the unpruned dense backward
# ----------------------------------------------------------------------------
def _dense_inputs(L):
    """fp64 views of a layer plus the rounded per-pair upstream gradients."""
    dt = L.dtype
    k = L.spec.k
    f = lambda arr: O.decode(arr, dt).astype(np.float64)
    w = L.topk_w.reshape(-1).astype(np.float32)
    t = np.arange(L.spec.P) // k
    grad = f(O.encode_rne(w[:, None] * O.decode(L.dY, dt)[t], dt))
    return grad, f(L.x), f(L.g), f(L.u), f(L.a), f(L.W_gu), f(L.W_down)


def rel_fro(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    d = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (d if d > 0 else 1.0)


@pytest.mark.parametrize("name,over", [("tiny", dict(quota="full")),
                                       ("qwen", dict(T=64, E=8, H=64, I=32, quota="full"))])
def test_t2_full_quota_equals_dense(name, over):
    L = small_layer(name, **over)
    r = O.pruned_backward(L)
    assert r["perm"].size == (L.topk_idx >= 0).sum()
    grad, x, g, u, a, Wgu, Wd = _dense_inputs(L)
    dWd, dWgu, dX = O.dense_backward(L.topk_idx, grad, x, g, u, a, Wgu, Wd)
    assert rel_fro(r["dW_down"], dWd) <= 1e-12
    assert rel_fro(r["dW_gu"], dWgu) <= 1e-12
    assert rel_fro(r["dX"], dX) <= 1e-12


# ----------------------------------------------------------------------------
# T4: dropped pairs contribute exactly zero
# ----------------------------------------------------------------------------
def test_t4_dropped_equals_dense_with_zero_weight():
    L = small_layer("tiny")
    r = O.pruned_backward(L)
    grad, x, g, u, a, Wgu, Wd = _dense_inputs(L)
    dropped = r["pos"] < 0
    grad[dropped] = 0.0
    dWd, dWgu, dX = O.dense_backward(L.topk_idx, grad, x, g, u, a, Wgu, Wd)
    assert rel_fro(r["dW_down"], dWd) <= 1e-12
    assert rel_fro(r["dW_gu"], dWgu) <= 1e-12
    assert rel_fro(r["dX"], dX) <= 1e-12


@pytest.mark.parametrize("name,over", [("tiny", {}), ("qwen", dict(T=128, E=8, H=64, I=32))])
def test_t4_dropped_rows_never_read(name, over):
    """NaN in the a, g, u rows of dropped pairs (after selection) changes nothing."""
    L = small_layer(name, **over)
    s = L.spec
    r = O.pruned_backward(L)
    dropped = np.nonzero(r["pos"] < 0)[0]
    nan = O.encode_rne(np.full((1, s.I), np.nan, np.float32), s.dtype)
    a2, g2, u2 = L.a.copy(), L.g.copy(), L.u.copy()
    a2[dropped] = nan
    g2[dropped] = nan
    u2[dropped] = nan
    Xp, DYp, Ap, Gp, Up = O.pack(r["perm"], L.topk_w, s.k, L.x, L.dY, a2, g2, u2, s.dtype)
    dWd, dWgu, dXp, _ = O.expert_backward(Xp, DYp, Ap, Gp, Up, r["offsets"], L.W_gu, L.W_down, s.dtype)
    dX = O.unpack(dXp, r["pos"], s.T, s.k)
    for got, ref in ((dWd, r["dW_down"]), (dWgu, r["dW_gu"]), (dX, r["dX"])):
        assert np.isfinite(got).all()
        np.testing.assert_array_equal(got, ref)


# ----------------------------------------------------------------------------
# T5: the dense backward equals finite differences of the forward
# ----------------------------------------------------------------------------
def test_t5_finite_differences():
    rng = np.random.default_rng(5)
    T, E, k, H, I = 5, 3, 2, 6, 4
    idx = np.array([[0, 1], [2, 0], [1, 1], [2, -1], [0, 2]], np.int32)
    w = rng.random((T, k))
    x = rng.standard_normal((T, H))
    Wgu = rng.standard_normal((E, 2 * I, H)) * 0.5
    Wd = rng.standard_normal((E, H, I)) * 0.5
    dY = rng.standard_normal((T, H))

    def loss(x_, Wgu_, Wd_):
        Y, *_ = O.forward(idx, w, x_, Wgu_, Wd_)
        return float((dY * Y).sum())

    _, g, u, a = O.forward(idx, w, x, Wgu, Wd)
    grad = (w.reshape(-1)[:, None] * dY[np.arange(T * k) // k])
    dWd, dWgu, dX = O.dense_backward(idx, grad, x, g, u, a, Wgu, Wd)

    h = 1e-6

    def fd(arr, setter):
        out = np.zeros_like(arr)
        for i in np.ndindex(arr.shape):
            plus, minus = arr.copy(), arr.copy()
            plus[i] += h
            minus[i] -= h
            out[i] = (setter(plus) - setter(minus)) / (2 * h)
        return out

    fd_Wd = fd(Wd, lambda v: loss(x, Wgu, v))
    fd_Wgu = fd(Wgu, lambda v: loss(x, v, Wd))
    fd_x = fd(x, lambda v: loss(v, Wgu, Wd))
    assert rel_fro(dWd, fd_Wd) < 1e-7
    assert rel_fro(dWgu, fd_Wgu) < 1e-7
    assert rel_fro(dX, fd_x) < 1e-7

    # the pruned path in fp64 at full quota gives the same gradients
    score = O.lrm_score_f64(idx, w, dY, a)
    quota = np.full(E, 99, np.int32)
    counts, kept, offsets, perm, pos, _ = O.select_quota(idx, score.astype(np.float32), quota, E)
    Xp, DYp, Ap, Gp, Up = O.pack(perm, w.astype(np.float32), k, x, dY, a, g, u, "f64")
    dWd2, dWgu2, dXp, _ = O.expert_backward(Xp, DYp, Ap, Gp, Up, offsets, Wgu, Wd, "f64")
    dX2 = O.unpack(dXp, pos, T, k)
    assert rel_fro(dWd2, fd_Wd) < 1e-7
    assert rel_fro(dWgu2, fd_Wgu) < 1e-7
    assert rel_fro(dX2, fd_x) < 1e-7


def test_swiglu_derivative_closed_form():
    """d/dg [silu(g) u] = u s (1 + g (1 - s)) against the central difference of silu."""
    g = np.linspace(-8, 8, 401)
    s = O.sigmoid64(g)
    h = 1e-6
    silu = lambda v: v / (1 + np.exp(-v))
    fd = (silu(g + h) - silu(g - h)) / (2 * h)
    np.testing.assert_allclose(s * (1 + g * (1 - s)), fd, rtol=1e-7, atol=1e-9)


def test_row_sampled_backward_matches_whole_expert_backward():
    """The per-row helpers used on full-size layers agree with the whole-expert path."""
    L = small_layer("qwen", T=96, E=8, H=64, I=32)
    s = L.spec
    r = O.pruned_backward(L)
    rows = np.arange(0, r["perm"].size, 3)
    dgu, dxp = O.expert_backward_rows(rows, r["offsets"], r["DYp"], r["Gp"], r["Up"], L.W_gu,
                                      L.W_down, s.dtype)
    for row in rows:
        np.testing.assert_allclose(dgu[int(row)], r["dGUp"][row], rtol=1e-13, atol=1e-300)
        np.testing.assert_allclose(dxp[int(row)], r["dXp"][row], rtol=1e-13, atol=1e-300)
    tokens = [0, 5, 17, 95]
    need = [int(p) for t in tokens for p in r["pos"].reshape(-1, s.k)[t] if p >= 0]
    _, dxp_all = O.expert_backward_rows(need, r["offsets"], r["DYp"], r["Gp"], r["Up"], L.W_gu,
                                        L.W_down, s.dtype)
    got = O.unpack_tokens(tokens, dxp_all, r["pos"], s.k, s.H)
    np.testing.assert_allclose(got, r["dX"][tokens], rtol=1e-12, atol=1e-300)


# ----------------------------------------------------------------------------
# quota controller
# ----------------------------------------------------------------------------
def test_quota_controller_reduces_to_the_capacity_rule():
    """No budget and cap = T*k/E gives the configs' capacity quotas (written independently)."""
    for name, over in (("qwen", dict(T=512, E=16, H=64, I=64)), ("glm", dict(T=384, E=8, H=64, I=64))):
        L = small_layer(name, **over)
        s = L.spec
        q, c = O.quota_controller(L.topk_idx, s.E, (s.T * s.k) // s.E, -1)
        np.testing.assert_array_equal(c, L.counts)
        np.testing.assert_array_equal(q, inputs.quota_from_counts(L.counts, s))


@pytest.mark.parametrize("seed", range(6))
def test_quota_controller_budget_properties(seed):
    """Within budget, never above count or cap, and maximal: one more level would not fit."""
    rng = np.random.default_rng(seed)
    E = int(rng.integers(1, 20))
    idx = rng.integers(-1, E + 2, size=(int(rng.integers(1, 300)), 3)).astype(np.int32)
    c = np.bincount(idx[(idx >= 0) & (idx < E)], minlength=E)
    cap = int(rng.integers(-1, 60))
    budget = int(rng.integers(-1, int(c.sum()) + 5))
    q, counts = O.quota_controller(idx, E, cap, budget)
    np.testing.assert_array_equal(counts, c)
    capped = c if cap <= 0 else np.minimum(c, cap)
    assert (q <= capped).all() and (q >= 0).all()
    if budget < 0 or capped.sum() <= budget:
        np.testing.assert_array_equal(q, capped)
        return
    assert q.sum() <= budget
    tau = q.max()
    assert (q == np.minimum(capped, tau)).all()
    assert np.minimum(capped, tau + 1).sum() > budget      # the next level would not fit


def test_quota_controller_worked_example():
    """counts (9, 5, 2, 0), budget 10 -> level 4 -> quotas (4, 4, 2, 0); with cap 3 -> (3, 3, 2, 0)."""
    idx = np.array([0] * 9 + [1] * 5 + [2] * 2, np.int32).reshape(-1, 1)
    q, c = O.quota_controller(idx, 4, 0, 10)
    assert c.tolist() == [9, 5, 2, 0] and q.tolist() == [4, 4, 2, 0]
    q, _ = O.quota_controller(idx, 4, 3, 10)
    assert q.tolist() == [3, 3, 2, 0]
    q, _ = O.quota_controller(idx, 4, 0, 0)
    assert q.tolist() == [0, 0, 0, 0]


# ----------------------------------------------------------------------------
# routing-weight gradient (reading R8)
# ----------------------------------------------------------------------------
def test_router_grad_equals_finite_differences_of_the_forward():
    """L(w) = sum_t <dY_t, Y_t(w)> with the fp64 forward; central differences in
    each routing weight give dL/dw_p, which must equal <dY_t, y_p>."""
    layer = small_layer("tiny", seed=4, T=6, E=3, H=16, I=8)
    s = layer.spec
    x = O.decode(layer.x, s.dtype).astype(np.float64)
    Wgu = O.decode(layer.W_gu, s.dtype).astype(np.float64)
    Wd = O.decode(layer.W_down, s.dtype).astype(np.float64)
    dY = O.decode(layer.dY, s.dtype).astype(np.float64)
    w = layer.topk_w.astype(np.float64)
    _, _, _, a = O.forward(layer.topk_idx, w, x, Wgu, Wd)
    y = np.zeros((s.P, s.H))
    for p in range(s.P):
        y[p] = Wd[layer.topk_idx.reshape(-1)[p]] @ a[p]
    dw, st = O.router_grad(layer.topk_idx, layer.dY, y.astype(np.float32), s.dtype, s.E)
    assert st == 0
    h = 1e-4
    for p in range(s.P):
        wp, wm = w.copy(), w.copy()
        wp.reshape(-1)[p] += h
        wm.reshape(-1)[p] -= h
        Lp = float((dY * O.forward(layer.topk_idx, wp, x, Wgu, Wd)[0]).sum())
        Lm = float((dY * O.forward(layer.topk_idx, wm, x, Wgu, Wd)[0]).sum())
        fd = (Lp - Lm) / (2 * h)
        assert abs(float(dw[p]) - fd) <= 1e-5 * max(1e-3, abs(fd)), (p, dw[p], fd)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_router_grad_dyadic_exact_and_masks(dtype):
    """Small multiples of 1/8 make every step exact: the canonical dot equals the
    fp64 dot bit for bit.  Empty, invalid and (with pos) dropped slots give +0."""
    rng = np.random.default_rng(7)
    T, k, E, H = 5, 3, 4, 64
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    idx[0, 1] = -1
    idx[2, 2] = E + 1
    dY = (rng.integers(-8, 9, size=(T, H)) / 8).astype(np.float32)
    y = (rng.integers(-8, 9, size=(T * k, H)) / 8).astype(np.float32)
    dw, st = O.router_grad(idx, O.encode_rne(dY, dtype), O.encode_rne(y, dtype), dtype, E)
    exact = (np.repeat(dY.astype(np.float64), k, axis=0) * y.astype(np.float64)).sum(axis=1)
    flat = idx.reshape(-1)
    for p in range(T * k):
        want = exact[p] if 0 <= flat[p] < E else 0.0
        assert float(dw[p]) == want and not (want == 0 and np.signbit(dw[p]))
    assert st == O.ST_BAD_EXPERT
    pos = np.arange(T * k, dtype=np.int32)
    pos[[3, 4, 9]] = -1
    dw2, _ = O.router_grad(idx, O.encode_rne(dY, dtype), O.encode_rne(y, dtype), dtype, E, pos=pos)
    assert float(dw2[3]) == 0.0 and float(dw2[4]) == 0.0 and float(dw2[9]) == 0.0
    keep = (pos >= 0)
    np.testing.assert_array_equal(dw2[keep].view(np.uint32), dw[keep].view(np.uint32))


def test_row_dot_of_a_row_with_itself_is_its_norm():
    """Two separately written loops agree bit for bit on x.x = ||x||^2 (so the
    hand-worked order pin of the norm also holds for the dot)."""
    x = np.random.default_rng(8).standard_normal((9, 8 * 40)).astype(np.float32)
    for vec in (4, 8):
        np.testing.assert_array_equal(O.row_dot(x, x, vec).view(np.uint32),
                                      O.row_sq_norm(x, vec).view(np.uint32))


# ----------------------------------------------------------------------------
# integer redistribution over expert copies (reading R11)
# ----------------------------------------------------------------------------
def _brute_force_peak(m, A):
    """Minimum over every integer plan of the peak load (tiny instances)."""
    import itertools
    E, G = A.shape
    per_expert = []
    for e in range(E):
        gs = [g for g in range(G) if A[e, g]]
        opts = []
        for split in itertools.product(range(m[e] + 1), repeat=len(gs)):
            if sum(split) == m[e]:
                row = [0] * G
                for g, c in zip(gs, split):
                    row[g] = c
                opts.append(row)
        per_expert.append(opts)
    best = None
    for plan in itertools.product(*per_expert):
        peak = max(sum(plan[e][g] for e in range(E)) for g in range(G))
        best = peak if best is None else min(best, peak)
    return best


@pytest.mark.parametrize("seed", range(12))
def test_redistribute_equals_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    E, G = int(rng.integers(1, 4)), int(rng.integers(1, 4))
    m = rng.integers(0, 5, size=E)
    A = rng.random((E, G)) < 0.6
    A[np.arange(E), rng.integers(0, G, size=E)] = True      # every expert has a copy
    x, L = O.redistribute(m, A)
    assert L == _brute_force_peak(m, A)
    assert np.array_equal(x.sum(axis=1), m) and np.all(x[~A] == 0) and np.all(x >= 0)
    assert x.sum(axis=0).max() == L if m.sum() else L == 0


def test_redistribute_closed_forms():
    # one copy per expert: the peak is the most loaded GPU's own experts
    A = np.eye(4, dtype=bool)[[0, 1, 1, 3, 2]]
    m = np.array([7, 2, 9, 4, 1])
    assert O.redistribute(m, A)[1] == 11
    # every expert everywhere: ceil(M / G)
    A = np.ones((5, 3), bool)
    assert O.redistribute(m, A)[1] == -(-23 // 3)
    # a hot expert with two copies next to cold single-copy experts
    A = np.zeros((3, 3), bool)
    A[0, [0, 1]] = True
    A[1, 1] = A[2, 2] = True
    assert O.redistribute([10, 4, 1], A)[1] == 7
    with pytest.raises(ValueError):
        O.redistribute([1, 0], np.array([[False, False], [True, True]]))


def test_split_by_destination_covers_each_global_run_once():
    """Two ranks' rows of the same experts, cut by one plan: every (copy, expert)
    run is filled exactly once, in global order, and each block keeps pair order."""
    plan = np.array([[3, 4, 0], [0, 2, 2], [5, 0, 0]])
    m0 = np.array([4, 1, 2])
    m1 = plan.sum(axis=1) - m0
    got = {}
    for rank, (mine, start) in enumerate([(m0, np.zeros(3)), (m1, m0)]):
        offsets = np.concatenate([[0], np.cumsum(mine)])
        perm = np.arange(offsets[-1]) * 10 + rank            # ascending within each expert
        pd, do, deo = O.split_by_destination(perm, offsets, plan, start)
        assert sorted(pd.tolist()) == sorted(perm.tolist())
        for g in range(3):
            for e in range(3):
                blk = pd[do[g] + deo[g, e]: do[g] + deo[g, e + 1]]
                assert list(blk) == sorted(blk)
                got.setdefault((g, e), 0)
                got[(g, e)] += len(blk)
    for g in range(3):
        for e in range(3):
            assert got[(g, e)] == plan[e, g]


def test_send_positions_put_each_row_back():
    """send_positions is the defining inverse of the split: the send slot of local
    packed row r holds that row's pair, and every slot is used once."""
    plan = np.array([[1, 3], [2, 0], [0, 4]])
    mine = np.array([3, 2, 3])
    offsets = np.concatenate([[0], np.cumsum(mine)])
    perm = np.array([5, 9, 14, 2, 30, 7, 11, 40])               # arbitrary pair ids
    start = np.array([1, 0, 1])
    pd, do, _ = O.split_by_destination(perm, offsets, plan, start)
    M = int(offsets[-1])
    rd = O.send_positions(perm, pd, M)
    assert sorted(rd.tolist()) == list(range(M))
    assert all(pd[rd[r]] == perm[r] for r in range(M))
    # one destination keeps the packed order: the map is the identity
    pd1, _, _ = O.split_by_destination(perm, offsets, mine.reshape(-1, 1) + start.reshape(-1, 1) * 0,
                                       None)
    assert O.send_positions(perm, pd1, M).tolist() == list(range(M))


def _group_by_sorting(tab):
    """Brute force for group_received: tag every received row with (expert, source,
    arrival index) and sort by that tag."""
    tab = np.asarray(tab)
    G, E = tab.shape[0], tab.shape[1] - 1
    tags, j = [], 0
    for q in range(G):
        for e in range(E):
            for i in range(tab[q, e], tab[q, e + 1]):
                tags.append((e, q, i, j))
                j += 1
    tags.sort()
    order = [t[3] for t in tags]
    counts = np.bincount([t[0] for t in tags], minlength=E) if tags else np.zeros(E, int)
    return order, np.concatenate([[0], np.cumsum(counts)])


def test_group_received_against_sorting_and_closed_forms():
    rng = np.random.default_rng(5)
    for G, E in ((1, 4), (3, 5), (4, 2), (2, 7)):
        cnt = rng.integers(0, 4, size=(G, E))
        cnt[0, 0] = 0                                       # empty blocks occur
        tab = np.concatenate([np.zeros((G, 1), int), np.cumsum(cnt, axis=1)], axis=1)
        order, inv, offs = O.group_received(tab)
        want_order, want_offs = _group_by_sorting(tab)
        assert order.tolist() == want_order
        assert offs.tolist() == list(want_offs)
        assert np.array_equal(inv[order], np.arange(len(order)))
        if G == 1:                                          # one source: already grouped
            assert order.tolist() == list(range(len(order)))
    # two sources, one expert each way: source 1's rows of expert 0 come before
    # source 0's rows of expert 1
    order, inv, offs = O.group_received([[0, 0, 2], [0, 1, 1]])
    assert order.tolist() == [2, 0, 1] and offs.tolist() == [0, 1, 3]


def test_pruned_backward_equals_torch_autograd_on_the_retained_pairs():
    """The pruned oracle equals torch autograd (fp64) of a forward that contains only
    the retained pairs: dropping a pair from the backward is the same as dropping
    its term from the layer output, for dW and for dX (library routine pin)."""
    layer = small_layer("qwen", seed=23, T=24, E=4, k=2, H=16, I=8, dtype="f32",
                        quota="half_ceil")
    s = layer.spec
    ref = O.pruned_backward(layer)
    keep = ref["pos"] >= 0
    x = torch.tensor(O.decode(layer.x, s.dtype), dtype=torch.float64, requires_grad=True)
    Wgu = torch.tensor(O.decode(layer.W_gu, s.dtype), dtype=torch.float64, requires_grad=True)
    Wd = torch.tensor(O.decode(layer.W_down, s.dtype), dtype=torch.float64, requires_grad=True)
    dY = torch.tensor(O.decode(layer.dY, s.dtype), dtype=torch.float64)
    w = torch.tensor(layer.topk_w, dtype=torch.float64)
    Y = torch.zeros(s.T, s.H, dtype=torch.float64)
    for t in range(s.T):
        for j in range(s.k):
            p = t * s.k + j
            if not keep[p]:
                continue
            e = int(layer.topk_idx[t, j])
            g = Wgu[e, : s.I] @ x[t]
            u = Wgu[e, s.I:] @ x[t]
            Y[t] = Y[t] + w[t, j] * (Wd[e] @ (torch.nn.functional.silu(g) * u))
    (dY * Y).sum().backward()
    # the oracle's packed gradient rows are fp32-rounded w * dY (storage f32):
    # compare at the fp32 rounding level of that one product
    assert rel_fro(ref["dW_down"], Wd.grad.numpy()) < 1e-6
    assert rel_fro(ref["dW_gu"], Wgu.grad.numpy()) < 1e-6
    assert rel_fro(ref["dX"], x.grad.numpy()) < 1e-6


# ----------------------------------------------------------------------------
# unpack in storage arithmetic (R12)
# ----------------------------------------------------------------------------
def _random_pos(rng, T, k, keep_frac):
    """pos[T*k]: each kept slot gets a distinct packed row, the rest -1."""
    keep = rng.random(T * k) < keep_frac
    pos = np.full(T * k, -1, np.int32)
    pos[keep] = rng.permutation(int(keep.sum())).astype(np.int32)
    return pos, int(keep.sum())


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_unpack_storage_exact_on_dyadic_inputs(dtype):
    """Multiples of 1/8 in [-1/2, 1/2]: every fp32 partial sum of up to 8 rows is
    exact and so is its bf16 rounding, so the result equals the fp64 return."""
    rng = np.random.default_rng(5)
    T, k, H = 37, 8, 24
    pos, M = _random_pos(rng, T, k, 0.4)
    vals = (rng.integers(-4, 5, size=(M, H)) / 8.0).astype(np.float32)
    stored = O.encode_rne(vals, dtype)
    got = O.decode(O.unpack_storage(stored, pos, T, k, dtype), dtype)
    want = O.unpack(vals.astype(np.float64), pos, T, k)
    np.testing.assert_array_equal(got.astype(np.float64), want)


def test_unpack_storage_sums_in_fp32_in_slot_order():
    """1 + 2^-24 rounds to 1 (tie to even) in fp32, twice; the small rows first,
    or an fp64 sum, would give 1 + 2^-23."""
    rows = np.array([[1.0], [2.0 ** -24], [2.0 ** -24]], np.float32)
    ascending = np.array([0, 1, 2], np.int32)
    small_first = np.array([1, 2, 0], np.int32)
    assert O.unpack_storage(rows, ascending, 1, 3, "f32")[0, 0] == np.float32(1.0)
    assert O.unpack_storage(rows, small_first, 1, 3, "f32")[0, 0] == np.float32(1 + 2.0 ** -23)


def test_unpack_storage_rounds_once_to_bf16():
    """1 + 2^-8 + 2^-8 = 1 + 2^-7 exactly in fp32, a bf16 value; rounding after
    each add would tie 1 + 2^-8 down to 1 and stay there."""
    rows = O.encode_rne(np.array([[1.0], [2.0 ** -8], [2.0 ** -8]], np.float32), "bf16")
    got = O.unpack_storage(rows, np.array([0, 1, 2], np.int32), 1, 3, "bf16")
    assert O.decode(got, "bf16")[0, 0] == np.float32(1 + 2.0 ** -7)


def test_unpack_storage_special_cases():
    """k = 1 copies the row; nothing retained gives +0 bits; -0 rows give +0."""
    rng = np.random.default_rng(6)
    rows = O.encode_rne(rng.standard_normal((5, 16)).astype(np.float32), "bf16")
    pos = np.array([3, -1, 0, 4, 1, 2], np.int32)
    got = O.unpack_storage(rows, pos, 6, 1, "bf16")
    for t, r in enumerate(pos):
        np.testing.assert_array_equal(got[t], rows[r] if r >= 0 else np.zeros(16, np.uint16))
    neg0 = np.full((1, 8), 0x8000, np.uint16)                 # bf16 -0.0
    assert not O.unpack_storage(neg0, np.array([0], np.int32), 1, 1, "bf16").any()
