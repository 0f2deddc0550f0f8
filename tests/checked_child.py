"""Child process of test_checked_gpu.py, run with LRMOE_CHECKED=1 so that the
binding loads the checked-index debug library (liblrmoe_checked.so).

1. The whole path on small layers (bf16 and fp32, ragged and tile-edge sizes)
   matches the oracle exactly as the normal build does, with status 0: the
   checks never fire on valid inputs.
2. Grouped GEMMs given offsets that break their contract (not rising, or ending
   past rows_cap) raise LRMOE_ST_BAD_INDEX and write nothing.  The operands are
   views into larger allocations, so even a kernel without the checks would stay
   inside memory the process owns.
Prints "checked ok" and exits 0 on success.
"""
from __future__ import annotations

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

LAYERS = {
    "qwen-mini": dict(name="qwen", T=512, E=8, k=4, H=256, I=192),
    "ragged": dict(name="qwen", T=300, E=6, k=3, H=320, I=136, quota="half_ceil"),
    "glm-mini": dict(name="glm", T=384, E=8, k=8, H=512, I=352, quota="keep:1/4"),
    "tiny-f32": dict(name="tiny"),
    "f32-ragged": dict(name="tiny", T=100, E=5, k=3, H=36, I=20),
    "one-expert": dict(name="qwen", T=200, E=1, k=1, H=64, I=64, quota="half_ceil"),
}


def bad_offsets_cases(L, torch, dtype):
    E, K, N, N2, full, cap = 4, 256, 192, 128, 1024, 512
    dev = "cuda"
    g = torch.Generator(device=dev).manual_seed(7)
    rows_full = torch.randn(full, K, device=dev, generator=g).to(dtype)
    W = torch.randn(E, K, N, device=dev, generator=g).to(dtype)
    in_full = torch.randn(full, N2, device=dev, generator=g).to(dtype)
    rows, in_rows = rows_full[:cap], in_full[:cap]  # rows_cap = cap
    for offs in ([0, 200, 400, 500, cap + 100], [0, 300, 200, 400, 500]):
        offsets = torch.tensor(offs, dtype=torch.int32, device=dev)
        st = torch.zeros(1, dtype=torch.int32, device=dev)
        out = torch.full((full, N), float("nan"), device=dev).to(dtype)
        L.lrmoe_grouped_dgrad(rows, W, offsets, L.LRMOE_EPI_STORE, out, status=st)
        dW = torch.full((E, K, N2), float("nan"), device=dev)
        st2 = torch.zeros(1, dtype=torch.int32, device=dev)
        L.lrmoe_grouped_wgrad(rows, in_rows, offsets, dW, status=st2)
        torch.cuda.synchronize()
        for what, s, t in (("dgrad", st, out), ("wgrad", st2, dW)):
            assert int(s.item()) & L.ST_BAD_INDEX, f"{dtype} {what} {offs}: no BAD_INDEX"
            assert bool(torch.isnan(t.float()).all()), f"{dtype} {what} {offs}: wrote output"


def main() -> int:
    import torch

    from oracle import lrmoe_oracle as O
    from pruned_expert_backward_lrmoe_b200 import inputs
    from pruned_expert_backward_lrmoe_b200 import lrmoe as L
    from tests import parity as PT

    assert L.LIB_PATH.endswith("liblrmoe_checked.so"), L.LIB_PATH
    L.load()
    with open("/proc/self/maps") as f:
        assert "liblrmoe_checked.so" in f.read(), "checked library not mapped"

    for key, kw in LAYERS.items():
        kw = dict(kw)
        layer = inputs.make_layer(inputs.spec(kw.pop("name"), **kw), seed=0)
        ref = O.pruned_backward(layer)
        for out, packed in ((PT.run_steps(layer), ("Xp", "DYp", "Ap", "Gp", "Up")),
                            (PT.run_chain(layer), PT.chain_packed(layer))):
            M = PT.check_selection(layer, out, ref)
            PT.check_pack(layer, out, ref, M, packed)
            PT.check_gradients(layer, out, ref)
            assert int(out["status"].item()) == 0, key
    bad_offsets_cases(L, torch, torch.bfloat16)
    bad_offsets_cases(L, torch, torch.float32)
    print("checked ok")
    return 0


if __name__ == "__main__":
    sys.exit(main())
