"""The redistributed multi-GPU backward of one MoE layer, built from the C ABI.

"LRMoE урезает обратный проход MoE ...", section "Что делает LRMoE", bullets 4-5:
after each rank has selected its own retained pairs, an integer plan spreads every
expert's retained pairs over the admissible copies of that expert (smallest peak
load, no new copies); the rows are grouped by receiver and expert and move in one
compact all-to-all; every copy runs the grouped GEMMs on what it received, and the
result returns to the original layout.

Every rank holds the weights of every expert (data-parallel copies); `admissible`
[E][G] says which ranks may compute which expert's pairs.  The weight gradients are
summed over ranks.  Collectives go through torch.distributed (NCCL on GPUs); every
data movement on the device is a library kernel (split, pack, gather, unpack).
Host syncs: the summed counts for the planner and the block sizes of the all-to-all.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch
import torch.distributed as dist

from . import lrmoe as L

_ROWS = ("Xp", "DYp", "Ap", "Gp", "Up")


def _world(group):
    if dist.is_available() and dist.is_initialized():
        return dist.get_rank(group), dist.get_world_size(group)
    return 0, 1


def _all_to_all_rows(out: torch.Tensor, inp: torch.Tensor, recv_rows, send_rows, group):
    if dist.is_available() and dist.is_initialized():
        dist.all_to_all_single(out, inp, list(recv_rows), list(send_rows), group=group)
    else:
        out.copy_(inp)


def redistributed_backward(inp: Dict[str, torch.Tensor], admissible: np.ndarray,
                           group=None, stats: Optional[dict] = None) -> Dict[str, torch.Tensor]:
    """This rank's tokens in `inp` (topk_idx, topk_w, quota, x, dY, g, u, a, W_gu,
    W_down); `admissible` [E][G] bool, G = world size.  Returns dW_down and dW_gu
    (summed over ranks) and this rank's dX, plus the selection outputs."""
    rank, world = _world(group)
    T, k = inp["topk_idx"].shape
    E, H, I = inp["W_down"].shape
    dev = inp["x"].device
    dt = inp["x"].dtype
    adm = np.asarray(admissible, bool)
    if adm.shape != (E, world):
        raise ValueError(f"admissible must be [E][G] = [{E}][{world}], got {adm.shape}")
    out = L.alloc_buffers(T, k, E, H, I, dt, device=dev)
    st = out["status"]
    st.zero_()

    # local selection
    L.lrmoe_score(inp["topk_idx"], inp["topk_w"], inp["dY"], inp["a"], E, out["score"], st)
    L.lrmoe_select_quota(inp["topk_idx"], out["score"], inp["quota"], out["counts"], out["kept"],
                         out["offsets"], out["perm"], out["pos"], out["workspace"], st)

    # summed counts -> plan; this rank's first global row of every expert
    kept = out["kept"].to(torch.int64)
    every = [torch.zeros_like(kept) for _ in range(world)]
    if world > 1:
        dist.all_gather(every, kept, group=group)
    else:
        every[0].copy_(kept)
    m = torch.stack(every).sum(0).cpu().numpy()
    start = torch.stack(every[:rank]).sum(0) if rank else torch.zeros_like(kept)
    plan, peak = L.lrmoe_redistribute(m, adm)

    # rows grouped by receiver and expert, gathered into the send buffer
    P = T * k
    perm_dest = torch.empty(P, dtype=torch.int32, device=dev)
    dest_off = torch.empty(world + 1, dtype=torch.int32, device=dev)
    dest_exp = torch.empty(world, E + 1, dtype=torch.int32, device=dev)
    L.lrmoe_split_by_destination(out["perm"], out["offsets"],
                                 torch.from_numpy(plan.astype(np.int32)).to(dev), perm_dest,
                                 dest_off, dest_exp, global_start=start.to(torch.int32), status=st)
    send = {n: torch.empty_like(out[n]) for n in _ROWS}
    L.lrmoe_pack(perm_dest, dest_off, inp["topk_w"], inp["x"], inp["dY"], inp["a"], inp["g"],
                 inp["u"], send["Xp"], send["DYp"], send["Ap"], send["Gp"], send["Up"], st)

    # block sizes, then the compact all-to-all of the rows
    tab_in = torch.empty_like(dest_exp)
    if world > 1:
        dist.all_to_all_single(tab_in.view(-1), dest_exp.view(-1), group=group)
    else:
        tab_in.copy_(dest_exp)
    send_rows = np.diff(dest_off.cpu().numpy()).astype(np.int64)
    tab = tab_in.cpu().numpy().astype(np.int64)          # [source][E+1] expert offsets
    recv_rows = tab[:, E]
    R = int(recv_rows.sum())
    recv = {}
    for n in _ROWS:
        buf = torch.empty(max(R, 1), send[n].shape[1], dtype=dt, device=dev)
        _all_to_all_rows(buf[:R], send[n][: int(send_rows.sum())], recv_rows, send_rows, group)
        recv[n] = buf

    # regroup by expert (sources in rank order) and run the grouped GEMMs
    base = np.concatenate([[0], np.cumsum(recv_rows)])
    order, offs = [], [0]
    for e in range(E):
        for q in range(world):
            order.extend(range(base[q] + tab[q, e], base[q] + tab[q, e + 1]))
        offs.append(len(order))
    order_d = torch.tensor(order, dtype=torch.int32, device=dev)
    offs_d = torch.tensor(offs, dtype=torch.int32, device=dev)
    mine = {n: torch.empty(max(R, 1), recv[n].shape[1], dtype=dt, device=dev) for n in _ROWS}
    for n in _ROWS:
        L.lrmoe_gather_rows(recv[n], order_d, mine[n], st)
    dGUp = torch.empty(max(R, 1), 2 * I, dtype=dt, device=dev)
    dXp_mine = torch.empty(max(R, 1), H, dtype=dt, device=dev)
    L.lrmoe_grouped_dgrad(mine["DYp"], inp["W_down"], offs_d, L.LRMOE_EPI_SWIGLU_BWD, dGUp,
                          Gp=mine["Gp"], Up=mine["Up"], status=st)
    L.lrmoe_grouped_wgrad(mine["DYp"], mine["Ap"], offs_d, out["dW_down"], status=st)
    L.lrmoe_grouped_wgrad(dGUp, mine["Xp"], offs_d, out["dW_gu"], status=st)
    L.lrmoe_grouped_dgrad(dGUp, inp["W_gu"], offs_d, L.LRMOE_EPI_STORE, dXp_mine, status=st)
    if world > 1:
        dist.all_reduce(out["dW_down"], group=group)
        dist.all_reduce(out["dW_gu"], group=group)

    # dX_p rows back to their source, into this rank's packed order, then unpacked
    inv = np.empty(len(order), np.int64)
    inv[np.asarray(order, np.int64)] = np.arange(len(order))
    back_src = torch.empty_like(dXp_mine)
    L.lrmoe_gather_rows(dXp_mine, torch.tensor(inv, dtype=torch.int32, device=dev), back_src, st)
    M = int(out["offsets"][-1].item())
    back = torch.empty(max(int(send_rows.sum()), 1), H, dtype=dt, device=dev)
    _all_to_all_rows(back[: int(send_rows.sum())], back_src[:R], send_rows, recv_rows, group)
    # local packed row r holds pair perm[r]; it came back at the position of that
    # pair in perm_dest
    pd = perm_dest[:M].cpu().numpy()
    where = np.empty(P, np.int64)
    where[pd] = np.arange(M)
    local_idx = where[out["perm"][:M].cpu().numpy()]
    L.lrmoe_gather_rows(back, torch.tensor(local_idx, dtype=torch.int32, device=dev),
                        out["dXp"], st)
    L.lrmoe_unpack(out["dXp"], out["pos"], T, k, out["dX"], st)
    if stats is not None:
        stats.update(peak=int(peak), plan=plan, sent=int(send_rows.sum() - send_rows[rank]),
                     received=int(R - recv_rows[rank]))
    return out
