"""Guard canaries: every buffer a C-ABI call is given sits between two sentinel
pages, and after the calls both pages (and every input) are unchanged.

Each guarded buffer is a view into a larger byte buffer filled with 0xA5: one
page before it, and after it the rest of its 256-byte rounding plus one page.
A kernel that writes a byte outside the buffer it was given (an off-by-one row,
a ragged-tail store, a stray index) changes a sentinel and fails the test, even
when the stray write lands in memory the process owns.  The results are still
checked against the oracle, so the guarded run is an ordinary parity run.

Shapes: the small edge cases (E = 1, k = 1, T < 32, fp32, ragged H/I, empty
experts) and an expert-size case around the 128- and 256-row tiles
(m_e = 127, 129, 255, 257 and 1).
"""
import math

import numpy as np
import pytest
import torch

from oracle import lrmoe_oracle as O
from pruned_expert_backward_lrmoe_b200 import inputs
from pruned_expert_backward_lrmoe_b200 import lrmoe as L
from tests import parity as PT

pytestmark = pytest.mark.gpu

PAGE = 4096
FILL = 0xA5


class Guard:
    """Device buffers with sentinel pages around each one."""

    def __init__(self):
        self.bufs = []

    def empty(self, shape, dtype):
        shape = tuple(shape)
        n = math.prod(shape) * torch.empty((), dtype=dtype).element_size()
        body = (n + 255) // 256 * 256
        raw = torch.full((PAGE + body + PAGE,), FILL, dtype=torch.uint8, device="cuda")
        self.bufs.append((raw, n))
        return raw[PAGE:PAGE + n].view(dtype).view(shape)

    def like(self, t):
        g = self.empty(t.shape, t.dtype)
        g.copy_(t)
        return g

    def check(self):
        torch.cuda.synchronize()
        for i, (raw, n) in enumerate(self.bufs):
            head, tail = raw[:PAGE], raw[PAGE + n:]
            assert bool((head == FILL).all()), f"buffer {i}: bytes before it were written"
            assert bool((tail == FILL).all()), f"buffer {i}: bytes after it were written"


def guarded_buffers(G, layer):
    s = layer.spec
    tdt = torch.bfloat16 if s.dtype == "bf16" else torch.float32
    proto = L.alloc_buffers(s.T, s.k, s.E, s.H, s.I, tdt)
    out = {k: G.empty(v.shape, v.dtype) for k, v in proto.items()}
    out["status"].zero_()
    return out


def tile_edge_layer():
    """Four experts that keep 127, 129, 255 and 257 pairs and one that keeps 1."""
    s = inputs.spec("qwen", T=512, E=5, k=4, H=192, I=136)
    rng = np.random.default_rng(5)
    idx = np.stack([rng.permutation(s.E)[: s.k] for _ in range(s.T)]).astype(np.int32)
    return inputs.make_layer(s, seed=5, topk_idx=idx,
                             quota=np.array([127, 129, 255, 257, 1], np.int32))


LAYERS = {
    "tiny-f32": lambda: inputs.make_layer(inputs.spec("tiny"), seed=0),
    "T17-E1-k1": lambda: inputs.make_layer(
        inputs.spec("qwen", T=17, E=1, k=1, H=64, I=64, quota="half_ceil"), seed=1),
    "ragged": lambda: inputs.make_layer(
        inputs.spec("qwen", T=300, E=6, k=3, H=320, I=136, quota="half_ceil"), seed=2),
    "f32-ragged": lambda: inputs.make_layer(inputs.spec("tiny", T=100, E=5, k=3, H=36, I=20),
                                            seed=3),
    "glm-mini-empty": lambda: inputs.make_layer(
        inputs.spec("glm", T=96, E=16, k=2, H=256, I=96, quota="keep:1/4"), seed=4),
    "tile-edges": tile_edge_layer,
}


def check_against_oracle(layer, out, ref, packed):
    M = PT.check_selection(layer, out, ref)
    PT.check_pack(layer, out, ref, M, packed)
    PT.check_gradients(layer, out, ref)
    assert int(out["status"].item()) == 0


@pytest.mark.parametrize("name", list(LAYERS))
def test_path_stays_inside_its_buffers(name):
    layer = LAYERS[name]()
    ref = O.pruned_backward(layer)
    G = Guard()
    plain = PT.device_inputs(layer)
    inp = {k: G.like(v) for k, v in plain.items()}

    out = PT.run_steps(layer, inp, poison=False, out=guarded_buffers(G, layer))
    check_against_oracle(layer, out, ref, ("Xp", "DYp", "Ap", "Gp", "Up"))
    out = PT.run_chain(layer, inp, out=guarded_buffers(G, layer))
    check_against_oracle(layer, out, ref, PT.chain_packed(layer))

    G.check()
    for k, v in plain.items():
        assert torch.equal(inp[k].view(torch.uint8), v.view(torch.uint8)), f"input {k} changed"


@pytest.mark.parametrize("name", ["ragged", "glm-mini-empty", "tile-edges"])
def test_other_entry_points_stay_inside_their_buffers(name):
    """Score from norms, router gradient, quota controller, the no-workspace
    selection, the exchange kernels (split by destination, wide rows, grouping of
    received rows, split of wide rows, row gather) and the opt-in GEMM variants."""
    layer = LAYERS[name]()
    s = layer.spec
    T, k, E, H, I, P = s.T, s.k, s.E, s.H, s.I, s.P
    G = Guard()
    plain = PT.device_inputs(layer)
    inp = {n: G.like(v) for n, v in plain.items()}
    i32 = torch.int32
    dt = inp["x"].dtype
    st = G.empty((1,), torch.int32)
    st.zero_()
    out = PT.run_chain(layer, inp, out=guarded_buffers(G, layer))
    torch.cuda.synchronize()
    M = int(out["offsets"][-1].item())

    norms = G.empty((P,), torch.float32)
    L.lrmoe_row_sqnorm(inp["a"].view(P, I), norms)
    score2 = G.empty((P,), torch.float32)
    L.lrmoe_score_from_norms(inp["topk_idx"], inp["topk_w"], inp["dY"], norms, E, score2, st)
    y = G.like(inp["x"].repeat_interleave(k, 0))  # a stand-in for the saved expert outputs
    dw = G.empty((P,), torch.float32)
    L.lrmoe_router_grad(inp["topk_idx"], inp["dY"], y, E, dw, pos=out["pos"], status=st)
    quota, counts = G.empty((E,), i32), G.empty((E,), i32)
    L.lrmoe_quota_controller(inp["topk_idx"], E, 64, P // 2, quota, counts, st)
    sel = {n: G.empty(out[n].shape, i32) for n in ("counts", "kept", "offsets", "perm", "pos")}
    L.lrmoe_select_quota_noalloc(inp["topk_idx"], out["score"], inp["quota"], sel["counts"],
                                 sel["kept"], sel["offsets"], sel["perm"], sel["pos"], st)

    # exchange kernels: two destinations (each expert's first half of rows to 0)
    kept = out["kept"].cpu().numpy().astype(np.int64)
    plan = np.stack([kept // 2, kept - kept // 2], 1).astype(np.int32)
    perm_dest, row_dest = G.empty((P,), i32), G.empty((P,), i32)
    dest_off, dest_exp = G.empty((3,), i32), G.empty((2, E + 1), i32)
    L.lrmoe_split_by_destination(out["perm"], out["offsets"], torch.from_numpy(plan).cuda(),
                                 perm_dest, dest_off, dest_exp, status=st, row_dest=row_dest)
    Wd = 2 * H + 3 * I
    wide = G.empty((P, Wd), dt)
    L.lrmoe_pack_wide(perm_dest, dest_off, inp["topk_w"], inp["x"], inp["dY"], inp["a"],
                      inp["g"], inp["u"], wide, st)
    Rc = max(M, 1)
    order, inv, offs = G.empty((Rc,), i32), G.empty((Rc,), i32), G.empty((E + 1,), i32)
    L.lrmoe_group_received(dest_exp, order, inv, offs, st)
    parts = {n: G.empty((Rc, H if n in ("Xp", "DYp") else I), dt)
             for n in ("Xp", "DYp", "Ap", "Gp", "Up")}
    L.lrmoe_split_wide(wide, order[:M], parts["Xp"], parts["DYp"], parts["Ap"], parts["Gp"],
                       parts["Up"], st)
    back = G.empty((Rc, H), dt)
    L.lrmoe_gather_rows(out["dXp"], inv[:M], back, st)

    # opt-in GEMM variants
    dGUp = G.empty((P, 2 * I), dt)
    L.lrmoe_grouped_dgrad_swiglu_gather(out["DYp"], inp["W_down"], out["offsets"], out["perm"],
                                        inp["g"].view(P, I), inp["u"].view(P, I), dGUp, st)
    dWgu = G.empty((E, 2 * I, H), torch.float32)
    L.lrmoe_grouped_wgrad_gather(out["dGUp"], out["perm"], inp["x"], k, P, out["offsets"], dWgu,
                                 status=st)
    dXp, dWd = G.empty((P, H), dt), G.empty((E, H, I), torch.float32)
    L.lrmoe_grouped_dgrad_wgrad(out["DYp"], inp["W_down"], out["offsets"], L.LRMOE_EPI_STORE,
                                G.empty((P, I), dt), out["Ap"], dWd, status=st)
    L.lrmoe_grouped_dgrad_wgrad(out["dGUp"], inp["W_gu"], out["offsets"], L.LRMOE_EPI_STORE, dXp,
                                out["Xp"], dWgu, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    # spot checks that the calls did their work (bit-exact ones from their own tests)
    assert torch.equal(score2.view(i32), out["score"].view(i32))
    for n in ("counts", "kept", "offsets", "pos"):
        assert torch.equal(sel[n], out[n]), n
    assert torch.equal(sel["perm"][:M], out["perm"][:M])
    assert torch.equal(dXp[:M].view(torch.int16), out["dXp"][:M].view(torch.int16))

    G.check()
    for n, v in plain.items():
        assert torch.equal(inp[n].view(torch.uint8), v.view(torch.uint8)), f"input {n} changed"
