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
data movement and every index map on the device is a library kernel (split, wide
pack, grouping of the received rows, split of the wide rows, gathers, unpack).
Host syncs: the summed counts for the planner and the block sizes of the
all-to-alls.
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


def redistributed_backward(inp: Dict[str, torch.Tensor], admissible: np.ndarray,
                           group=None, stats: Optional[dict] = None) -> Dict[str, torch.Tensor]:
    """This rank's tokens in `inp` (topk_idx, topk_w, quota, x, dY, g, u, a, W_gu,
    W_down); `admissible` [E][G] bool, G = world size.  Returns dW_down and dW_gu
    (summed over ranks) and this rank's dX, plus the selection outputs.

    Collectives, in order: all-gather of the retained counts, all-to-all of the
    per-destination expert tables, one all-to-all of the exchange rows, one
    all-reduce of both weight gradients, one all-to-all of the returned dX_p rows.
    Host synchronisations: the summed counts (the planner runs on the host) and
    the block sizes of the row all-to-alls; every index map is built on the device."""
    rank, world = _world(group)
    T, k = inp["topk_idx"].shape
    E, H, I = inp["W_down"].shape
    P = T * k
    dev = inp["x"].device
    dt = inp["x"].dtype
    adm = np.asarray(admissible, bool)
    if adm.shape != (E, world):
        raise ValueError(f"admissible must be [E][G] = [{E}][{world}], got {adm.shape}")
    out = L.alloc_buffers(T, k, E, H, I, dt, device=dev)
    # both weight gradients in one buffer, so that one all-reduce sums them
    dW = torch.empty(E * H * I + E * 2 * I * H, dtype=torch.float32, device=dev)
    out["dW_down"] = dW[: E * H * I].view(E, H, I)
    out["dW_gu"] = dW[E * H * I:].view(E, 2 * I, H)
    st = out["status"]
    st.zero_()
    i32 = dict(dtype=torch.int32, device=dev)

    # local selection
    L.lrmoe_score(inp["topk_idx"], inp["topk_w"], inp["dY"], inp["a"], E, out["score"], st)
    L.lrmoe_select_quota(inp["topk_idx"], out["score"], inp["quota"], out["counts"], out["kept"],
                         out["offsets"], out["perm"], out["pos"], out["workspace"], st)

    # summed counts -> plan (host sync 1); this rank's first global row of every expert
    kept = out["kept"].to(torch.int64)
    every = [torch.zeros_like(kept) for _ in range(world)]
    if world > 1:
        dist.all_gather(every, kept, group=group)
    else:
        every[0].copy_(kept)
    m = torch.stack(every).sum(0).cpu().numpy()
    start = torch.stack(every[:rank]).sum(0) if rank else torch.zeros_like(kept)
    plan, peak = L.lrmoe_redistribute(m, adm)

    # rows grouped by receiver and expert, packed as exchange rows [x | w dY | a | g | u]
    perm_dest = torch.empty(P, **i32)
    dest_off = torch.empty(world + 1, **i32)
    dest_exp = torch.empty(world, E + 1, **i32)
    row_dest = torch.empty(P, **i32)
    L.lrmoe_split_by_destination(out["perm"], out["offsets"],
                                 torch.from_numpy(plan.astype(np.int32)).to(dev), perm_dest,
                                 dest_off, dest_exp, global_start=start.to(torch.int32), status=st,
                                 row_dest=row_dest)
    Wd = 2 * H + 3 * I
    send = torch.empty(P, Wd, dtype=dt, device=dev)
    L.lrmoe_pack_wide(perm_dest, dest_off, inp["topk_w"], inp["x"], inp["dY"], inp["a"], inp["g"],
                      inp["u"], send, st)

    # every receiver learns its expert tables; block sizes to the host (sync 2)
    tab_in = torch.empty_like(dest_exp)
    if world > 1:
        dist.all_to_all_single(tab_in.view(-1), dest_exp.view(-1), group=group)
    else:
        tab_in.copy_(dest_exp)
    sizes = torch.cat([dest_off[1:] - dest_off[:-1], tab_in[:, E]]).cpu().numpy().astype(np.int64)
    send_rows, recv_rows = sizes[:world], sizes[world:]
    S, R = int(send_rows.sum()), int(recv_rows.sum())

    # one all-to-all moves all five operands of every exchanged pair
    recv = torch.empty(max(R, 1), Wd, dtype=dt, device=dev)
    if world > 1:
        dist.all_to_all_single(recv[:R], send[:S], recv_rows.tolist(), send_rows.tolist(),
                               group=group)
    else:
        recv[:R].copy_(send[:S])

    # the receiver's dense per-expert blocks, built on the device
    Rc = max(R, 1)
    order = torch.empty(Rc, **i32)
    inv = torch.empty(Rc, **i32)
    offs = torch.empty(E + 1, **i32)
    L.lrmoe_group_received(tab_in, order, inv, offs, st)
    mine = {n: torch.empty(Rc, H if n in ("Xp", "DYp") else I, dtype=dt, device=dev)
            for n in _ROWS}
    L.lrmoe_split_wide(recv, order[:R], mine["Xp"], mine["DYp"], mine["Ap"], mine["Gp"],
                       mine["Up"], st)
    dGUp = torch.empty(Rc, 2 * I, dtype=dt, device=dev)
    dXp_mine = torch.empty(Rc, H, dtype=dt, device=dev)
    L.lrmoe_grouped_dgrad(mine["DYp"], inp["W_down"], offs, L.LRMOE_EPI_SWIGLU_BWD, dGUp,
                          Gp=mine["Gp"], Up=mine["Up"], status=st)
    L.lrmoe_grouped_wgrad(mine["DYp"], mine["Ap"], offs, out["dW_down"], status=st)
    L.lrmoe_grouped_wgrad(dGUp, mine["Xp"], offs, out["dW_gu"], status=st)
    L.lrmoe_grouped_dgrad(dGUp, inp["W_gu"], offs, L.LRMOE_EPI_STORE, dXp_mine, status=st)
    if world > 1:
        dist.all_reduce(dW, group=group)

    # dX_p rows: grouped -> arrival order, back to their sources (send order), then
    # each to its local packed row, then unpacked
    back_src = torch.empty(Rc, H, dtype=dt, device=dev)
    L.lrmoe_gather_rows(dXp_mine, inv[:R], back_src, st)
    back = torch.empty(max(S, 1), H, dtype=dt, device=dev)
    if world > 1:
        dist.all_to_all_single(back[:S], back_src[:R], send_rows.tolist(), recv_rows.tolist(),
                               group=group)
    else:
        back[:S].copy_(back_src[:R])
    L.lrmoe_gather_rows(back, row_dest[:S], out["dXp"], st)
    L.lrmoe_unpack(out["dXp"], out["pos"], T, k, out["dX"], st)
    if stats is not None:
        stats.update(peak=int(peak), plan=plan, sent=int(S - send_rows[rank]),
                     received=int(R - recv_rows[rank]))
    return out
