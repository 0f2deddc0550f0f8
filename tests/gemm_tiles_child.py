"""Child process of test_gemm_tiles_gpu.py: runs the whole path on a few small
bf16 layers and saves dW_down, dW_gu and dX to an .npz file (argv[1]).  The parent
runs it once with the default (two-SM) grouped-GEMM tiles and once with
LRMOE_GEMM_ONE_SM=1 (the environment is read once per process)."""
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
    "skew-mini": dict(name="skew", T=1024, E=16, k=4, H=128, I=128),
    "max-sizes": dict(name="qwen", T=512, E=1024, k=32, H=64, I=64),
}


def main() -> int:
    import numpy as np
    import torch

    from pruned_expert_backward_lrmoe_b200 import inputs
    from tests import parity as PT

    out = {}
    for key, kw in LAYERS.items():
        kw = dict(kw)
        layer = inputs.make_layer(inputs.spec(kw.pop("name"), **kw), seed=0)
        res = PT.run_chain(layer)
        assert int(res["status"].item()) == 0, key
        for n in ("dW_down", "dW_gu", "dX"):
            out[f"{key}/{n}"] = res[n].float().cpu().numpy()
    np.savez(sys.argv[1], **out)
    torch.cuda.synchronize()
    print("saved", len(out))
    return 0


if __name__ == "__main__":
    sys.exit(main())
