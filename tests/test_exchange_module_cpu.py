"""exchange.redistributed_backward's own multi-rank code on 2 and 3 gloo ranks
(CPU): every library device call is replaced by an oracle-backed CPU stand-in, so
what runs is the module's bookkeeping (summed counts, plan, global starts, split,
send slots, exchange rows, block sizes, the compact all-to-all, regrouping, one
dW reduction, the return and unpack of dX_p).  Each rank's dX and the summed dW must equal what each rank
computes from its own pairs alone."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
T_PER_RANK, E, K, H, I = 40, 5, 2, 16, 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _install_cpu_stand_ins(L, O, dtype):
    """Oracle-backed CPU versions of the library's device calls (fp32 storage)."""
    import torch

    def np32(t):
        return t.detach().cpu().numpy()

    def score(idx, w, dY, a, E_, out, status=None, stream=None):
        s, _ = O.lrm_score(np32(idx), np32(w), np32(dY), np32(a), dtype, E_)
        out.copy_(torch.from_numpy(s))

    def select(idx, sc, quota, counts, kept, offsets, perm, pos, ws, status=None, stream=None):
        c, k_, o, p, q, _ = O.select_quota(np32(idx), np32(sc), np32(quota), quota.numel())
        counts.copy_(torch.from_numpy(c.astype(np.int32)))
        kept.copy_(torch.from_numpy(k_.astype(np.int32)))
        offsets.copy_(torch.from_numpy(o.astype(np.int32)))
        perm.fill_(-7)
        perm[: len(p)] = torch.from_numpy(p.astype(np.int32))
        pos.copy_(torch.from_numpy(q.astype(np.int32)))

    def split(perm, offsets, plan, pd, do, deo, global_start=None, status=None, stream=None,
              row_dest=None):
        start = None if global_start is None else np32(global_start)
        a, b, c = O.split_by_destination(np32(perm), np32(offsets), np32(plan), start)
        pd[: len(a)] = torch.from_numpy(a)
        do.copy_(torch.from_numpy(b))
        deo.copy_(torch.from_numpy(c))
        if row_dest is not None:
            M = int(offsets[-1])
            row_dest[:M] = torch.from_numpy(O.send_positions(np32(perm), a, M))

    def pack_wide(perm, offsets, w, x, dY, a, g, u, rows, status=None, stream=None):
        M = int(offsets[-1])
        k_ = w.shape[1]
        parts = O.pack(np32(perm)[:M], np32(w), k_, np32(x), np32(dY), np32(a), np32(g), np32(u),
                       dtype)
        rows[:M] = torch.from_numpy(np.concatenate([np.asarray(r, np.float32) for r in parts],
                                                   axis=1))

    def group_received(tab, order, inv, offsets, status=None, stream=None):
        o, i, off = O.group_received(np32(tab))
        order[: len(o)] = torch.from_numpy(o)
        inv[: len(i)] = torch.from_numpy(i)
        offsets.copy_(torch.from_numpy(off))

    def split_wide(rows, idx, Xp, DYp, Ap, Gp, Up, status=None, stream=None):
        n = idx.numel()
        H_, I_ = Xp.shape[1], Ap.shape[1]
        src = rows[idx.long()]
        cols = np.cumsum([0, H_, H_, I_, I_, I_])
        for j, dst in enumerate((Xp, DYp, Ap, Gp, Up)):
            dst[:n] = src[:, cols[j]:cols[j + 1]]

    def gather(src, idx, dst, status=None, stream=None):
        if idx.numel():
            dst[: idx.numel()] = src[idx.long()]

    def dgrad(rows, W, offsets, epi, out, Gp=None, Up=None, status=None, stream=None):
        off = np32(offsets)
        r64, W64 = np32(rows).astype(np.float64), np32(W).astype(np.float64)
        for e in range(W.shape[0]):
            lo, hi = off[e], off[e + 1]
            if hi == lo:
                continue
            d = r64[lo:hi] @ W64[e]
            if epi == L.LRMOE_EPI_SWIGLU_BWD:
                g, u = np32(Gp)[lo:hi].astype(np.float64), np32(Up)[lo:hi].astype(np.float64)
                sg = O.sigmoid64(g)
                d = np.concatenate([d * u * sg * (1 + g * (1 - sg)), d * g * sg], axis=1)
            out[lo:hi] = torch.from_numpy(d.astype(np.float32))

    def wgrad(grad, inr, offsets, dW, accumulate=False, status=None, stream=None):
        off = np32(offsets)
        g64, i64 = np32(grad).astype(np.float64), np32(inr).astype(np.float64)
        out = np.zeros(dW.shape)
        for e in range(dW.shape[0]):
            out[e] = g64[off[e]:off[e + 1]].T @ i64[off[e]:off[e + 1]]
        dW.copy_(torch.from_numpy(out.astype(np.float32)))

    def unpack(dXp, pos, T, k_, dX, status=None, stream=None):
        dX.copy_(torch.from_numpy(O.unpack(np32(dXp).astype(np.float64), np32(pos), T, k_)
                                  .astype(np.float32)))

    L.lrmoe_score, L.lrmoe_select_quota = score, select
    L.lrmoe_split_by_destination, L.lrmoe_pack_wide, L.lrmoe_gather_rows = split, pack_wide, gather
    L.lrmoe_group_received, L.lrmoe_split_wide = group_received, split_wide
    L.lrmoe_grouped_dgrad, L.lrmoe_grouped_wgrad, L.lrmoe_unpack = dgrad, wgrad, unpack


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from oracle import lrmoe_oracle as O
    from pruned_expert_backward_lrmoe_b200 import exchange as X
    from pruned_expert_backward_lrmoe_b200 import inputs
    from pruned_expert_backward_lrmoe_b200 import lrmoe as L
    dist.init_process_group("gloo", rank=rank, world_size=world)
    _install_cpu_stand_ins(L, O, "f32")
    layer = inputs.make_layer(inputs.spec("tiny", T=world * T_PER_RANK, E=E, k=K, H=H, I=I),
                              seed=41)
    t0, t1 = rank * T_PER_RANK, (rank + 1) * T_PER_RANK
    sl = slice(t0 * K, t1 * K)
    mine = dict(topk_idx=layer.topk_idx[t0:t1], topk_w=layer.topk_w[t0:t1], x=layer.x[t0:t1],
                dY=layer.dY[t0:t1], a=layer.a[sl], g=layer.g[sl], u=layer.u[sl])
    flat = mine["topk_idx"].reshape(-1)
    counts = np.bincount(flat[(flat >= 0) & (flat < E)], minlength=E)
    mine["quota"] = inputs.quota_from_counts(counts, layer.spec).astype(np.int32)
    inp = {n: torch.from_numpy(np.ascontiguousarray(v)) for n, v in mine.items()}
    inp["W_gu"] = torch.from_numpy(np.ascontiguousarray(layer.W_gu))
    inp["W_down"] = torch.from_numpy(np.ascontiguousarray(layer.W_down))
    A = np.zeros((E, world), bool)
    A[np.arange(E), np.arange(E) % world] = True
    A[0, :] = True                                   # the hottest expert everywhere
    stats = {}
    out = X.redistributed_backward(inp, A, stats=stats)

    # reference: this rank's own pairs, alone
    sc, _ = O.lrm_score(mine["topk_idx"], mine["topk_w"], mine["dY"], mine["a"], "f32", E)
    _, _, offsets, perm, pos, _ = O.select_quota(mine["topk_idx"], sc, mine["quota"], E)
    rows = O.pack(perm, mine["topk_w"], K, mine["x"], mine["dY"], mine["a"], mine["g"],
                  mine["u"], "f32")
    dWd, dWgu, dXp, _ = O.expert_backward(*rows, offsets, layer.W_gu, layer.W_down, "f32")
    dX = O.unpack(dXp, pos, T_PER_RANK, K)
    results[rank] = dict(dX_err=float(np.abs(out["dX"].numpy() - dX).max() /
                                      max(1e-30, np.abs(dX).max())),
                         dWd=out["dW_down"].numpy(), dWgu=out["dW_gu"].numpy(),
                         ref_dWd=dWd, ref_dWgu=dWgu, sent=stats["sent"], peak=stats["peak"])
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_module_on_gloo_ranks(world):
    port = _free_port()
    with mp.Manager() as man:
        results = man.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        got = dict(results)
    assert set(got) == set(range(world))
    for r in range(world):
        assert got[r]["dX_err"] <= 1e-6                 # fp32 storage of dGU_p, dX_p
    for name in ("dWd", "dWgu"):
        ref = sum(got[r]["ref_" + name] for r in range(world))
        for r in range(world):
            assert np.abs(got[r][name] - ref).max() <= 1e-5 * np.abs(ref).max()
    assert sum(got[r]["sent"] for r in range(world)) > 0
    assert len({got[r]["peak"] for r in range(world)}) == 1
