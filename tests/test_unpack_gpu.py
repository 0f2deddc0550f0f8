"""a5 alone, bit for bit: lrmoe_unpack on seeded dX_p rows against the oracle's
return in storage arithmetic (fp32 sum in ascending slot order, one rounding).
Shapes span one and several 32-vector column chunks, ragged chunk tails, k = 1
and k = 32 with every slot retained, tokens with nothing retained, bf16
overflow to Inf, -0 rows, out-of-range rows, and the qwen-sized launch."""
import numpy as np
import pytest
import torch

from oracle import lrmoe_oracle as O
from pruned_expert_backward_lrmoe_b200 import lrmoe as L

pytestmark = pytest.mark.gpu

TORCH = {"bf16": torch.bfloat16, "f32": torch.float32}


def _pos(rng, T, k, keep_frac):
    keep = rng.random(T * k) < keep_frac
    pos = np.full(T * k, -1, np.int32)
    pos[keep] = rng.permutation(int(keep.sum())).astype(np.int32)
    return pos, int(keep.sum())


def _bits(t):
    return t.cpu().view(torch.int16 if t.dtype == torch.bfloat16 else torch.int32).numpy()


def _run(rows, pos, T, k, dtype, rows_cap=None):
    """rows: storage array [M, H] (uint16 bf16 bits or float32)."""
    M, H = rows.shape
    cap = rows_cap if rows_cap is not None else max(M, 1)
    dev = torch.zeros((cap, H), dtype=TORCH[dtype], device="cuda")
    if M:
        src = torch.from_numpy(rows.view(np.int16) if dtype == "bf16" else rows)
        dev[:M].copy_(src.view(TORCH[dtype]) if dtype == "bf16" else src)
    d_pos = torch.from_numpy(pos).cuda()
    dX = torch.full((T, H), float("nan"), dtype=TORCH[dtype], device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.lrmoe_unpack(dev, d_pos, T, k, dX, st)
    torch.cuda.synchronize()
    return dX, int(st.item())


def _want_bits(rows, pos, T, k, dtype):
    want = O.unpack_storage(rows, pos, T, k, dtype)
    return want.view(np.int16) if dtype == "bf16" else np.asarray(want, np.float32).view(np.int32)


@pytest.mark.parametrize("dtype,T,k,H,keep", [
    ("bf16", 1000, 8, 2048, 0.31),    # one 256-vector row: 8 chunks per lane group
    ("bf16", 333, 8, 4096, 0.5),      # 16 chunks
    ("bf16", 129, 32, 320, 1.0),      # k = 32, every slot retained, 40 vectors (ragged chunk)
    ("bf16", 64, 1, 8, 0.5),          # one vector per row, k = 1
    ("bf16", 77, 4, 8 * 33 * 8, 0.9), # 264 vectors: a ragged ninth chunk
    ("f32", 255, 2, 64, 0.6),         # the fp32 path, 16 vectors
    ("f32", 100, 4, 1028, 0.7),       # 257 vectors
    ("bf16", 50, 8, 2048, 0.0),       # nothing retained anywhere
])
def test_unpack_bit_exact(dtype, T, k, H, keep):
    rng = np.random.default_rng(T * 131 + k)
    pos, M = _pos(rng, T, k, keep)
    rows = O.encode_rne(rng.standard_normal((M, H)).astype(np.float32), dtype)
    dX, st = _run(rows, pos, T, k, dtype)
    assert st == 0
    np.testing.assert_array_equal(_bits(dX), _want_bits(rows, pos, T, k, dtype))


def test_unpack_qwen_sized_launch():
    """The benchmark's launch: T = 8192 tokens, top-8, H = 2048, about 31 % retained."""
    rng = np.random.default_rng(8192)
    T, k, H = 8192, 8, 2048
    pos, M = _pos(rng, T, k, 0.31)
    rows = O.encode_rne((0.01 * rng.standard_normal((M, H))).astype(np.float32), "bf16")
    dX, st = _run(rows, pos, T, k, "bf16")
    assert st == 0
    np.testing.assert_array_equal(_bits(dX), _want_bits(rows, pos, T, k, "bf16"))


def test_unpack_overflow_negative_zero_and_bad_rows():
    """The bf16 maximum 2^128 - 2^120 plus 1.5 * 2^119 is 2^128 - 2^118: exact and
    finite in fp32, above the midpoint to 2^128, so its one rounding gives Inf; a
    lone -0 row gives +0; rows at or past rows_cap are flagged and skipped."""
    T, k, H = 4, 3, 16
    vals = np.zeros((5, H), np.float32)
    vals[0] = np.float32(2.0 ** 128 - 2.0 ** 120)
    vals[1] = np.float32(1.5 * 2.0 ** 119)
    vals[2] = -0.0
    vals[3] = 1.5
    vals[4] = -2.25
    rows = O.encode_rne(vals, "bf16")
    pos = np.array([0, 1, -1,     # Inf after the bf16 rounding only
                    2, -1, -1,    # -0 alone
                    3, 9, 4,      # row 9 >= rows_cap: flagged, skipped
                    -1, -1, -1], np.int32)
    dX, st = _run(rows, pos, T, k, "bf16", rows_cap=5)
    assert st & L.ST_BAD_INDEX
    ok = pos.copy()
    ok[ok >= 5] = -1
    np.testing.assert_array_equal(_bits(dX), _want_bits(rows, ok, T, k, "bf16"))
    got = dX.float().cpu().numpy()
    assert np.isinf(got[0]).all() and not got[1].any() and not got[3].any()
