"""The pages' multi-GPU path on two gloo ranks (CPU), end to end, with the
oracle's arithmetic and the library's host planner: each rank selects its own
pairs, the counts are summed, the integer plan spreads every expert's retained
pairs over its copies, each rank splits its packed rows by receiver, a compact
all-to-all moves them, every copy runs the expert backward on what it received,
the weight gradients are summed over copies, and the dX_p rows travel back and
are unpacked.  The result must equal each rank computing its own pairs alone."""
import os
import socket
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
T_PER_RANK, E, K, H, I = 48, 4, 2, 16, 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_slice(layer, r):
    t0, t1 = r * T_PER_RANK, (r + 1) * T_PER_RANK
    sl = slice(t0 * K, t1 * K)
    return dict(idx=layer.topk_idx[t0:t1], w=layer.topk_w[t0:t1], x=layer.x[t0:t1],
                dY=layer.dY[t0:t1], a=layer.a[sl], g=layer.g[sl], u=layer.u[sl])


def _local(O, inputs, layer, d):
    s = layer.spec
    score, _ = O.lrm_score(d["idx"], d["w"], d["dY"], d["a"], s.dtype, E)
    flat = d["idx"].reshape(-1)
    counts = np.bincount(flat[(flat >= 0) & (flat < E)], minlength=E)
    quota = inputs.quota_from_counts(counts, s)
    _, kept, offsets, perm, pos, _ = O.select_quota(d["idx"], score, quota, E)
    return kept, offsets, perm, pos


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from oracle import lrmoe_oracle as O
    from pruned_expert_backward_lrmoe_b200 import inputs
    from pruned_expert_backward_lrmoe_b200 import lrmoe as L
    dist.init_process_group("gloo", rank=rank, world_size=world)
    layer = inputs.make_layer(inputs.spec("tiny", T=world * T_PER_RANK, E=E, k=K, H=H, I=I),
                              seed=31)
    s = layer.spec
    d = _rank_slice(layer, rank)
    kept, offsets, perm, pos = _local(O, inputs, layer, d)

    # reference: this rank's pairs on their own
    ref_p = O.pack(perm, d["w"], K, d["x"], d["dY"], d["a"], d["g"], d["u"], s.dtype)
    ref_dWd, ref_dWgu, ref_dXp, _ = O.expert_backward(*ref_p, offsets, layer.W_gu, layer.W_down,
                                                      s.dtype)
    ref_dX = O.unpack(ref_dXp, pos, T_PER_RANK, K)

    # global counts, copies, plan
    kt = torch.from_numpy(kept.astype(np.int64))
    m = kt.clone()
    dist.all_reduce(m)
    every = [torch.zeros_like(kt) for _ in range(world)]
    dist.all_gather(every, kt)
    start = sum(every[q] for q in range(rank)) if rank else torch.zeros_like(kt)
    A = np.zeros((E, world), bool)
    A[np.arange(E), np.arange(E) % world] = True
    A[int(np.argmax(m.numpy())), :] = True          # the hottest expert has a copy everywhere
    plan, peak = L.lrmoe_redistribute(m.numpy(), A)
    assert peak == O.redistribute_peak(m.numpy(), A)

    # split by receiver, pack the send buffer, compact all-to-all
    pd, do, deo = O.split_by_destination(perm, offsets, plan, start.numpy())
    send = [np.asarray(v, np.float64) for v in
            O.pack(pd, d["w"], K, d["x"], d["dY"], d["a"], d["g"], d["u"], s.dtype)]
    send_rows = np.diff(do).tolist()
    tab = torch.from_numpy(deo.astype(np.int64)).reshape(-1)
    tab_in = torch.empty_like(tab)
    dist.all_to_all_single(tab_in, tab, [E + 1] * world, [E + 1] * world)
    tab_in = tab_in.reshape(world, E + 1).numpy()          # per source: expert offsets
    recv_rows = tab_in[:, E].tolist()
    recv = []
    for arr in send:
        out = torch.empty((sum(recv_rows), arr.shape[1]), dtype=torch.float64)
        dist.all_to_all_single(out, torch.from_numpy(arr), recv_rows, send_rows)
        recv.append(out.numpy())
    # regroup by expert (sources in rank order), run the copy's expert backward
    src_base = np.concatenate([[0], np.cumsum(recv_rows)])
    order, offs = [], [0]
    for e in range(E):
        for q in range(world):
            order.extend(range(src_base[q] + tab_in[q, e], src_base[q] + tab_in[q, e + 1]))
        offs.append(len(order))
    order = np.asarray(order, np.int64)
    mine = [r[order].astype(np.float32) for r in recv]
    dWd, dWgu, dXp_mine, _ = O.expert_backward(*mine, np.asarray(offs), layer.W_gu,
                                               layer.W_down, s.dtype)
    served = np.asarray(offs[1:]) - np.asarray(offs[:-1])
    assert served.sum() == plan[:, rank].sum() and max(plan.sum(axis=0)) == peak
    # weight gradients: sum over copies; dX_p rows back to their source
    dWd_t, dWgu_t = torch.from_numpy(dWd), torch.from_numpy(dWgu)
    dist.all_reduce(dWd_t)
    dist.all_reduce(dWgu_t)
    back_recv_order = np.empty_like(dXp_mine)
    back_recv_order[order] = dXp_mine
    back = torch.empty((int(do[-1]), H), dtype=torch.float64)
    dist.all_to_all_single(back, torch.from_numpy(back_recv_order), send_rows, recv_rows)
    dXp_local = np.zeros((int(offsets[-1]), H))
    dXp_local[pos[pd]] = back.numpy()
    dX = O.unpack(dXp_local, pos, T_PER_RANK, K)
    results[rank] = dict(
        dX=float(np.abs(dX - ref_dX).max() / max(1e-30, np.abs(ref_dX).max())),
        dWd=dWd_t.numpy(), dWgu=dWgu_t.numpy(), ref_dWd=ref_dWd, ref_dWgu=ref_dWgu,
        moved=int(sum(send_rows) - send_rows[rank]))
    dist.destroy_process_group()


def test_two_ranks_redistribute_exchange_and_return():
    world = 2
    port = _free_port()
    with mp.Manager() as man:
        results = man.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        got = dict(results)
    assert set(got) == {0, 1}
    for r in range(world):
        assert got[r]["dX"] <= 1e-12
    for name in ("dWd", "dWgu"):
        ref = got[0]["ref_" + name] + got[1]["ref_" + name]
        for r in range(world):
            assert np.abs(got[r][name] - ref).max() <= 1e-12 * np.abs(ref).max()
    assert got[0]["moved"] + got[1]["moved"] > 0      # rows really crossed ranks
