"""Row norms and the score from saved norms on the GPU against the oracle, bit
for bit: ragged row counts, rows longer than one chunk, non-finite rows,
invalid expert ids, and the score buffer used in place as the norm input."""
import numpy as np
import pytest
import torch

from oracle import lrmoe_oracle as O
from pruned_expert_backward_lrmoe_b200 import inputs
from pruned_expert_backward_lrmoe_b200 import lrmoe as L
from tests.parity import storage_tensor as _device_rows

pytestmark = pytest.mark.gpu


def _rows(n, D, dtype, seed, special=False):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((n, D)) * rng.uniform(0.01, 3.0, size=(n, 1))).astype(np.float32)
    if special and n >= 4:
        x[1, :] = 0.0
        x[2, D // 2] = np.inf
        x[3, 0] = np.nan
    return O.encode_rne(x, dtype)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("n,D", [(1, 8), (7, 64), (1001, 768), (300, 1408), (129, 2048),
                                 (33, 4096), (5, 8200)])
def test_row_sqnorm_bit_exact(dtype, n, D):
    if dtype == "f32" and D % 4:
        pytest.skip("f32 rows are multiples of 4")
    enc = _rows(n, D, dtype, seed=n + D, special=True)
    ref = O.row_sq_norm(O.decode(enc, dtype), O.VEC[dtype])
    out = torch.full((n,), -7.0, device="cuda")
    L.lrmoe_row_sqnorm(_device_rows(enc, dtype), out)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    # a NaN row gives a NaN norm; its payload is not specified (the score
    # canonicalises NaN), every other value must match bit for bit
    nan = np.isnan(ref)
    np.testing.assert_array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_row_sqnorm_order_example(dtype):
    vec = O.VEC[dtype]
    x = np.zeros((2, 32 * vec), np.float32)
    x[:, 0], x[:, vec], x[:, 3 * vec] = 4096.0, 1.0, 1.0
    out = torch.zeros(2, device="cuda")
    L.lrmoe_row_sqnorm(_device_rows(O.encode_rne(x, dtype), dtype), out)
    torch.cuda.synchronize()
    assert out.tolist() == [16777218.0, 16777218.0]


@pytest.mark.parametrize("name,over", [("qwen", dict(T=1000, E=16, H=2048, I=768)),
                                       ("glm", dict(T=333, E=8, H=4096, I=1408)),
                                       ("tiny", dict(T=77))])
@pytest.mark.parametrize("in_place", [False, True])
def test_score_from_norms_bit_exact(name, over, in_place):
    layer = inputs.make_layer(inputs.spec(name, **over), seed=5)
    s = layer.spec
    idx = layer.topk_idx.copy()
    idx[3, 0] = s.E + 2          # invalid expert id: +0 and a status bit
    idx[4, 1] = -1               # empty slot
    dY = layer.dY.copy()
    n_a = O.row_sq_norm(O.decode(layer.a, s.dtype), O.VEC[s.dtype])
    n_a[5 * s.k] = np.float32(np.inf)
    n_a[6 * s.k + 1] = np.float32(np.nan)
    ref, st_ref = O.lrm_score_from_norms(idx, layer.topk_w, dY, n_a, s.dtype, s.E)
    d_idx = torch.from_numpy(idx).cuda()
    d_w = torch.from_numpy(layer.topk_w).cuda()
    d_dy = _device_rows(dY, s.dtype)
    d_na = torch.from_numpy(n_a).cuda()
    score = d_na if in_place else torch.full((s.P,), -7.0, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.lrmoe_score_from_norms(d_idx, d_w, d_dy, d_na, s.E, score, st)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(score.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    assert int(st.item()) == st_ref


def test_score_equals_norms_then_score_from_norms():
    layer = inputs.make_layer(inputs.spec("qwen", T=512, E=16, H=256, I=768), seed=6)
    s = layer.spec
    d_idx = torch.from_numpy(layer.topk_idx).cuda()
    d_w = torch.from_numpy(layer.topk_w).cuda()
    d_dy = _device_rows(layer.dY, s.dtype)
    d_a = _device_rows(layer.a, s.dtype)
    s1 = torch.empty(s.P, device="cuda")
    L.lrmoe_score(d_idx, d_w, d_dy, d_a, s.E, s1)
    na = torch.empty(s.P, device="cuda")
    L.lrmoe_row_sqnorm(d_a, na)
    s2 = torch.empty(s.P, device="cuda")
    L.lrmoe_score_from_norms(d_idx, d_w, d_dy, na, s.E, s2)
    torch.cuda.synchronize()
    assert torch.equal(s1.view(torch.int32), s2.view(torch.int32))
