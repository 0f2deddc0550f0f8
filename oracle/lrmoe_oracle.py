"""CPU oracle for the LRMoE pruned MoE expert backward -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously-correct numpy restatement of what the hot path computes.
Only the tests, the package smoke check and the benchmark's CPU-baseline leg may
import it; the product path never does.  It shares no code with the CUDA
library (only the seeded input generator, which holds none of this arithmetic).

Source of the method: the three news pages on LRMoE.  Citations name the page
title and section:
  [RU-B]  "LRMoE урезает обратный проход MoE ...", section "Что делает LRMoE:
          полный прямой проход, обрезанный обратный" (bullets 1-5 and the note
          after them); [FR-B] is the same section of the French page
          ("Ce que fait LRMoE : passe avant complète, passe arrière élaguée").
  [RU-C]  same page, section "Что показали эксперименты и где подвох".
  [DE]    "LRMoE führt eine Nachkalibrierung der Last ...", paragraphs 3-4.

What each function follows
--------------------------
lrm_score        [RU-B] bullet 3 / [FR-B] bullet 3 / [DE] para 3: a pair's
                 contribution to the expert weight update is the outer product
                 of the incoming gradient (w * dY) and the saved projection
                 input a; its squared Frobenius norm factorises into
                 w^2 * ||dY||^2 * ||a||^2, so no gradient matrix is formed.
select_quota     [RU-B] bullet 3 (last sentence) / [DE] para 3: within the
                 per-expert quota the pairs with the highest score stay.
pack             [RU-B] bullet 5 / [DE] para 4: retained gradient and
                 activation rows are gathered into dense per-expert blocks;
                 [RU-B] note: masking rows inside full tensors gives nothing,
                 only physically smaller matrices do.
expert_backward  [RU-B] bullet 5: variable-size grouped GEMMs on those blocks
                 with no zero padding (here: plain fp64 matmuls per expert).
unpack           [RU-B] bullet 5, last sentence: the result goes back to the
                 original layout.
unpack_storage   the same return in the storage arithmetic the device uses
                 (R12): fp32 sum in ascending slot order, one rounding.
dense_backward   the ordinary unpruned SwiGLU MoE expert backward (textbook
                 calculus); used only to pin the pruned functions.
forward          the ordinary SwiGLU MoE forward in fp64, used only by the
                 finite-difference pin ([RU-B] bullet 1: the forward stays full).
lrm_score_from_norms  the score with ||a_p||^2 given (saved by the forward);
                 the same three factors, multiplied in the same order.
redistribute     [RU-B] bullet 4 / [FR-B] bullet 4: the remaining pairs of each
                 expert are spread over the admissible copies of that expert
                 by an integer algorithm that minimises the peak load of one
                 GPU; no new copies appear (R11).
split_by_destination  [RU-B] bullet 5: retained rows are grouped by receiver
                 and expert, so the all-to-all moves compact blocks.
send_positions   where each local packed row sits in that send order (the map
                 that puts returned rows back in the local packed layout).
group_received   the receiver's side of [RU-B] bullet 5: rows that arrived from
                 every source, regrouped into one dense block per expert.
router_grad      the gradient of the routing weights, dL/dw_p = <dY_t, y_p>
                 with y_p = W_down[e] a_p the pair's expert output (the layer
                 output is sum_j w_tj y_tj); the pages do not treat it (R8).

Readings where the pages are silent:
  R1  "saved projection input" = a = silu(g)*u, the input of the down
      projection, because the incoming gradient there is w*dY.
  R2  one retained set serves dW_down, dW_gate, dW_up and dX.
  R3  canonical fp32 score order (below) so that selection is bit-comparable.
  R4  key = (score bits descending, pair index ascending); blocks in ascending
      expert id, rows inside a block in ascending pair index; NaN scores are
      canonicalised to 0x7FFFFFFF (rank above +Inf).
  R5  quotas are integers given as input; m_e = min(max(q_e, 0), c_e).
  R6  the packed gradient row is RNE_storage(fp32(w) * fp32(dY_t)); all
      gradient arithmetic afterwards is fp64 here.
  R7  topk_idx < 0 = not routed; idx >= E = invalid (skipped, status bit).
  R11 the load of a GPU is the number of retained pairs it serves (every pair of
      a layer costs the same); an expert's pairs, in the global order (source
      rank, then packed row), are cut into consecutive runs, one per copy in
      ascending GPU order, with the run lengths of the optimal plan.
  R8  the routing-weight gradient is not part of the pruned path; when asked
      for, it is <dY_t, y_p> with y_p saved by the forward, for every routed
      pair, or for the retained pairs only when pos is given (dropped pairs
      then get 0), in the canonical order below with x*x replaced by dY*y.
  R12 returning dX_p to the token layout sums a token's retained rows in fp32,
      starting from +0, in ascending slot order, and rounds once to the
      storage dtype; a token with nothing retained gets +0.

Canonical score order (R3), for one row v of D = V * VEC elements
(VEC = 8 for bf16 storage, 4 for fp32):
  1. 32 fp32 partials start at +0.  Partial l takes vectors c = l, l+32, ...
  2. inside a vector, elements in index order: acc = fl(acc + fl(x*x))
     (two RNE roundings, no fused multiply-add).
  3. butterfly: for o in 16, 8, 4, 2, 1: acc[l] = fl(acc[l] + acc[l ^ o]).
  4. the norm is acc[0].
  score = fl(fl(fl(w*w) * n_dY) * n_a).

Parity with the pages themselves is unpinned for R1 and R2 (the pages print no
worked example); every function below is pinned to closed forms, brute force,
library routines or finite differences by the tests under tests/.
"""
from __future__ import annotations

import numpy as np

ST_BAD_EXPERT = 1
ST_BAD_QUOTA = 2
ST_NONFINITE = 4

NAN_SCORE_BITS = np.uint32(0x7FFFFFFF)
VEC = {"bf16": 8, "f32": 4}


# ----------------------------------------------------------------------------
# storage helpers (bf16 kept as uint16 bit patterns)
# ----------------------------------------------------------------------------
def decode(arr: np.ndarray, dtype: str) -> np.ndarray:
    """Storage values -> float32.  bf16 bits b are the upper half of an fp32."""
    if dtype == "bf16":
        return (arr.astype(np.uint32) << np.uint32(16)).view(np.float32)
    if dtype in ("f32", "f64"):
        return np.asarray(arr)
    raise ValueError(dtype)


def encode_rne(v32: np.ndarray, dtype: str) -> np.ndarray:
    """float32 -> storage dtype with round-to-nearest-even; NaN -> 0x7FFF (bf16)."""
    if dtype in ("f32", "f64"):
        return np.asarray(v32)
    bits = np.ascontiguousarray(v32, dtype=np.float32).view(np.uint32)
    lsb = (bits >> np.uint32(16)) & np.uint32(1)
    rounded = (bits.astype(np.uint64) + np.uint64(0x7FFF) + lsb.astype(np.uint64)) >> np.uint64(16)
    out = rounded.astype(np.uint16)
    out[np.isnan(v32)] = np.uint16(0x7FFF)
    return out


# ----------------------------------------------------------------------------
# a1: LRM score
# ----------------------------------------------------------------------------
def row_sq_norm(rows32: np.ndarray, vec: int) -> np.ndarray:
    """Squared L2 norm of each row in the canonical fp32 order (R3)."""
    rows32 = np.ascontiguousarray(rows32, dtype=np.float32)
    n, D = rows32.shape
    assert D % vec == 0
    V = D // vec
    v = rows32.reshape(n, V, vec)
    acc = np.zeros((n, 32), dtype=np.float32)
    for r in range(0, V, 32):             # round r: lane l holds vector r + l
        nl = min(32, V - r)
        for j in range(vec):
            x = v[:, r:r + nl, j]
            acc[:, :nl] = acc[:, :nl] + x * x
    lane = np.arange(32)
    for o in (16, 8, 4, 2, 1):
        acc = acc + acc[:, lane ^ o]
    return acc[:, 0].copy()


def row_dot(rows_a32: np.ndarray, rows_b32: np.ndarray, vec: int) -> np.ndarray:
    """Row-wise dot products in the canonical order: 32 lane partials over
    vectors, fl(acc + fl(x*y)) element by element, then the butterfly."""
    A = np.ascontiguousarray(rows_a32, dtype=np.float32)
    B = np.ascontiguousarray(rows_b32, dtype=np.float32)
    n, D = A.shape
    assert B.shape == (n, D) and D % vec == 0
    V = D // vec
    va, vb = A.reshape(n, V, vec), B.reshape(n, V, vec)
    acc = np.zeros((n, 32), dtype=np.float32)
    with np.errstate(invalid="ignore", over="ignore"):
        for r in range(0, V, 32):
            nl = min(32, V - r)
            for j in range(vec):
                acc[:, :nl] = acc[:, :nl] + va[:, r:r + nl, j] * vb[:, r:r + nl, j]
        lane = np.arange(32)
        for o in (16, 8, 4, 2, 1):
            acc = acc + acc[:, lane ^ o]
    return acc[:, 0].copy()


def lrm_score(topk_idx, topk_w, dY, a, dtype: str, E: int):
    """score[p] = w_p^2 * ||dY_t||^2 * ||a_p||^2 for every routed pair p = t*k + j.

    Non-routed (idx < 0) and invalid (idx >= E) slots get +0 and are never
    selected; invalid ones set ST_BAD_EXPERT.  NaN scores set ST_NONFINITE.
    """
    n_a = row_sq_norm(decode(a, dtype), VEC[dtype])            # [P]
    return lrm_score_from_norms(topk_idx, topk_w, dY, n_a, dtype, E)


def lrm_score_from_norms(topk_idx, topk_w, dY, a_sqnorm, dtype: str, E: int):
    """The same score with ||a_p||^2 given (saved by the forward): the three
    factors of the factorisation, multiplied in the canonical order."""
    T, k = topk_idx.shape
    idx = topk_idx.reshape(-1)
    w = topk_w.reshape(-1).astype(np.float32)
    status = 0
    if np.any(idx >= E):
        status |= ST_BAD_EXPERT
    routed = (idx >= 0) & (idx < E)
    n_dy = row_sq_norm(decode(dY, dtype), VEC[dtype])          # [T]
    n_a = np.asarray(a_sqnorm, dtype=np.float32).reshape(-1)
    n_dy_p = np.repeat(n_dy, k)
    with np.errstate(invalid="ignore", over="ignore"):
        s = ((w * w) * n_dy_p) * n_a
    s = np.where(routed, s, np.float32(0.0)).astype(np.float32)
    bits = s.view(np.uint32).copy()
    nan = np.isnan(s)
    if np.any(nan):
        status |= ST_NONFINITE
        bits[nan] = NAN_SCORE_BITS
    if np.any(np.isinf(s)):
        status |= ST_NONFINITE
    return bits.view(np.float32), status


def lrm_score_f64(topk_idx, topk_w, dY64, a64):
    """Same factorised score in fp64 (no canonical order); used by pins only."""
    T, k = topk_idx.shape
    w = topk_w.reshape(-1).astype(np.float64)
    n_dy = np.repeat((dY64.astype(np.float64) ** 2).sum(1), k)
    n_a = (a64.astype(np.float64) ** 2).sum(1)
    return w * w * n_dy * n_a


# ----------------------------------------------------------------------------
# quota controller (before the backward)
# ----------------------------------------------------------------------------
def router_grad(topk_idx, dY, y, dtype: str, E: int, pos=None):
    """dw[p] = <dY_t, y_p> for routed pairs (R8); +0 for empty and invalid slots
    and, when pos is given, for pairs with pos[p] < 0.  Invalid ids set
    ST_BAD_EXPERT.  y [T*k, H] is the pair's saved expert output."""
    T, k = topk_idx.shape
    idx = topk_idx.reshape(-1)
    status = ST_BAD_EXPERT if np.any(idx >= E) else 0
    keep = (idx >= 0) & (idx < E)
    if pos is not None:
        keep &= np.asarray(pos).reshape(-1) >= 0
    dy_p = np.repeat(decode(dY, dtype), k, axis=0)
    d = row_dot(dy_p, decode(y, dtype), VEC[dtype])
    return np.where(keep, d, np.float32(0.0)).astype(np.float32), status


def redistribute_peak(m, admissible):
    """Smallest achievable peak load, from Hall's condition for the transportation
    problem: the plan with peak L exists iff for every set S of GPUs the experts
    whose copies all lie in S fit, sum_{e: A_e within S} m_e <= L |S|.  So
    L* = max over nonempty S of ceil(D(S) / |S|).  Exponential in G (small G only)."""
    m = np.asarray(m, np.int64)
    A = np.asarray(admissible, bool)
    E, G = A.shape
    best = 0
    for mask in range(1, 1 << G):
        inside = np.array([(mask >> g) & 1 for g in range(G)], bool)
        confined = ~np.any(A & ~inside[None, :], axis=1) & np.any(A, axis=1)
        D = int(m[confined].sum())
        size = int(inside.sum())
        best = max(best, -(-D // size))
    return best


def redistribute(m, admissible):
    """Integer plan x[e][g] >= 0: sum_g x[e][g] = m_e, x[e][g] = 0 where expert e
    has no copy on GPU g, and max_g sum_e x[e][g] equal to redistribute_peak.
    The plan comes from augmenting paths (breadth-first, Edmonds-Karp) on the
    network source -> expert (cap m_e) -> its copies -> sink (cap L*)."""
    m = np.asarray(m, np.int64)
    A = np.asarray(admissible, bool)
    E, G = A.shape
    if np.any((m > 0) & ~np.any(A, axis=1)):
        raise ValueError("an expert with retained pairs has no copy")
    L = redistribute_peak(m, A)
    n = E + G + 2
    src, snk = E + G, E + G + 1
    cap = np.zeros((n, n), np.int64)
    for e in range(E):
        cap[src, e] = m[e]
        for g in range(G):
            if A[e, g]:
                cap[e, E + g] = m[e]
    for g in range(G):
        cap[E + g, snk] = L
    flow = np.zeros((n, n), np.int64)
    while True:
        prev = [-1] * n
        prev[src] = src
        queue = [src]
        for u in queue:
            for v in range(n):
                if prev[v] < 0 and cap[u, v] - flow[u, v] > 0:
                    prev[v] = u
                    queue.append(v)
        if prev[snk] < 0:
            break
        push, v = None, snk
        while v != src:
            u = prev[v]
            r = cap[u, v] - flow[u, v]
            push = r if push is None else min(push, r)
            v = u
        v = snk
        while v != src:
            u = prev[v]
            flow[u, v] += push
            flow[v, u] -= push
            v = u
    x = np.zeros((E, G), np.int64)
    for e in range(E):
        for g in range(G):
            x[e, g] = max(0, flow[e, E + g])
    assert np.array_equal(x.sum(axis=1), m), "no plan at the Hall peak"
    return x, L


def split_by_destination(perm, offsets, plan, global_start=None):
    """Regroup this rank's packed rows by destination GPU, then expert (R11).

    Expert e's local rows r in [offsets[e], offsets[e+1]) have global indices
    global_start[e] + (r - offsets[e]); copy g serves the global run
    [C[e][g], C[e][g+1]) with C the prefix sum of plan[e] over g.  Returns
    perm_dest (pair ids in destination-major order), dest_offsets [G+1] and
    dest_expert_offsets [G][E+1] (offsets inside each destination's block)."""
    plan = np.asarray(plan, np.int64)
    E, G = plan.shape
    offsets = np.asarray(offsets, np.int64)
    start = np.zeros(E, np.int64) if global_start is None else np.asarray(global_start, np.int64)
    C = np.concatenate([np.zeros((E, 1), np.int64), np.cumsum(plan, axis=1)], axis=1)
    blocks = [[[] for _ in range(E)] for _ in range(G)]
    for e in range(E):
        for r in range(offsets[e], offsets[e + 1]):
            gi = start[e] + (r - offsets[e])
            for g in range(G):
                if C[e, g] <= gi < C[e, g + 1]:
                    blocks[g][e].append(int(perm[r]))
                    break
            else:
                raise ValueError("plan does not cover every retained row")
    perm_dest, dest_offsets = [], [0]
    dest_expert_offsets = np.zeros((G, E + 1), np.int32)
    for g in range(G):
        for e in range(E):
            dest_expert_offsets[g, e + 1] = dest_expert_offsets[g, e] + len(blocks[g][e])
            perm_dest.extend(blocks[g][e])
        dest_offsets.append(len(perm_dest))
    return (np.asarray(perm_dest, np.int32), np.asarray(dest_offsets, np.int32),
            dest_expert_offsets)


def send_positions(perm, perm_dest, M: int):
    """Slot of each local packed row r < M in the destination-major send order of
    split_by_destination: the i with perm_dest[i] = perm[r] (a pair id occurs
    once).  The returned rows come back in send order, and this map puts each
    one back at its local packed row."""
    where = {}
    for i in range(M):
        where[int(perm_dest[i])] = i
    return np.asarray([where[int(perm[r])] for r in range(M)], np.int32)


def group_received(src_expert_offsets):
    """Regroup received rows expert-major ([RU-B] bullet 5: the receiving copy runs
    the grouped GEMMs on dense per-expert blocks).

    The received rows are source-major: source q's block follows the blocks of
    sources 0..q-1 and holds its rows of expert e at [T[q][e], T[q][e+1]) inside
    the block (T = src_expert_offsets [G][E+1], each source's dest_expert_offsets
    row for this receiver).  Grouped order: experts ascending, inside an expert
    the sources in rank order, inside a source the arrival order.  Returns order
    (grouped position i holds received row order[i]), inv (its inverse) and the
    grouped offsets [E+1]."""
    tab = np.asarray(src_expert_offsets, np.int64)
    G, E = tab.shape[0], tab.shape[1] - 1
    base = [0]
    for q in range(G):
        base.append(base[-1] + int(tab[q, E]))
    order, offsets = [], [0]
    for e in range(E):
        for q in range(G):
            order.extend(range(base[q] + int(tab[q, e]), base[q] + int(tab[q, e + 1])))
        offsets.append(len(order))
    inv = [0] * len(order)
    for i, j in enumerate(order):
        inv[j] = i
    return (np.asarray(order, np.int32), np.asarray(inv, np.int32),
            np.asarray(offsets, np.int32))


def quota_controller(topk_idx, E: int, cap: int, max_pairs: int):
    """Per-expert quotas from routed counts, a per-expert cap and a pair budget.

    [RU-B] bullet 2: before the backward a controller sees how many tokens came to
    each expert and, within memory limits, fixes how many pairs of each expert stay
    for the whole layer call.  Reading (water-filling): q_e = min(c_e, cap, tau) with
    tau the largest integer level for which sum_e q_e <= max_pairs, so the most
    loaded experts are cut first.  cap <= 0: no per-expert cap; max_pairs < 0: no
    budget.  Returns (quota[E] int32, counts[E] int32).
    """
    idx = np.asarray(topk_idx).reshape(-1)
    counts = np.zeros(E, dtype=np.int64)
    for e in idx:
        if 0 <= e < E:
            counts[e] += 1
    capped = counts.copy() if cap <= 0 else np.minimum(counts, cap)
    if max_pairs < 0 or capped.sum() <= max_pairs:
        return capped.astype(np.int32), counts.astype(np.int32)
    tau = 0
    for level in range(int(capped.max()) + 1):     # largest level within the budget
        if np.minimum(capped, level).sum() <= max_pairs:
            tau = level
    return np.minimum(capped, tau).astype(np.int32), counts.astype(np.int32)


# ----------------------------------------------------------------------------
# a2: per-expert top-quota selection
# ----------------------------------------------------------------------------
def select_quota(topk_idx, score, quota, E: int):
    """Keep, per expert, the m_e = min(max(q_e,0), c_e) pairs with the largest key.

    Returns counts[E], kept[E], offsets[E+1], perm[M], pos[P], status.
    perm lists the retained pairs, expert blocks in ascending e and pairs in
    ascending index inside a block; pos[p] is p's packed row or -1.
    """
    idx = topk_idx.reshape(-1)
    P = idx.size
    bits = np.ascontiguousarray(score, dtype=np.float32).view(np.uint32)
    quota = np.asarray(quota, dtype=np.int64)
    status = 0
    if np.any(quota < 0):
        status |= ST_BAD_QUOTA
    if np.any(idx >= E):
        status |= ST_BAD_EXPERT
    counts = np.zeros(E, dtype=np.int32)
    kept = np.zeros(E, dtype=np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    pos = np.full(P, -1, dtype=np.int32)
    blocks = []
    for e in range(E):
        pairs = np.nonzero(idx == e)[0]                        # ascending p
        c = pairs.size
        m = int(min(max(int(quota[e]), 0), c))
        counts[e] = c
        kept[e] = m
        offsets[e + 1] = offsets[e] + m
        # sort by (bits descending, p ascending); lexsort keys: last is primary
        order = np.lexsort((pairs, np.uint32(0xFFFFFFFF) - bits[pairs]))
        chosen = np.sort(pairs[order[:m]])
        blocks.append(chosen)
    perm = np.concatenate(blocks).astype(np.int32) if blocks else np.zeros(0, np.int32)
    pos[perm] = np.arange(perm.size, dtype=np.int32)
    return counts, kept, offsets, perm, pos, status


# ----------------------------------------------------------------------------
# a3: physical compaction
# ----------------------------------------------------------------------------
def pack(perm, topk_w, k: int, x, dY, a, g, u, dtype: str):
    """Gather retained rows into dense blocks (storage dtype).

    X_p[r] = x[t], DY_p[r] = RNE(fp32(w_p) * fp32(dY[t])), A_p/G_p/U_p[r] = a/g/u[p],
    with p = perm[r], t = p // k.
    """
    perm = np.asarray(perm, dtype=np.int64)
    t = perm // k
    w = topk_w.reshape(-1)[perm].astype(np.float32)
    if dtype == "f64":
        DYp = w.astype(np.float64)[:, None] * dY[t]
    else:
        DYp = encode_rne(w[:, None] * decode(dY, dtype)[t], dtype)
    return x[t].copy(), DYp, a[perm].copy(), g[perm].copy(), u[perm].copy()


# ----------------------------------------------------------------------------
# a4: expert backward on the compacted blocks
# ----------------------------------------------------------------------------
def sigmoid64(g):
    return 1.0 / (1.0 + np.exp(-g))


def expert_backward(Xp, DYp, Ap, Gp, Up, offsets, W_gu, W_down, dtype: str, experts=None):
    """fp64 SwiGLU expert backward over each expert's packed rows.

    For rows R_e = [offsets[e], offsets[e+1]):
      dA      = DY_p W_down[e]                      (m_e x I)
      dG      = dA * u * s * (1 + g (1 - s)),  s = sigmoid(g)
      dU      = dA * g * s
      dW_down = DY_p^T A_p                          (H x I)
      dW_gu   = [dG | dU]^T X_p                     (2I x H)
      dX_p    = [dG | dU] W_gu[e]                   (m_e x H)
    Returns (dW_down [E,H,I] or dict, dW_gu, dXp [M,H], dGUp [M,2I]) in fp64.
    `experts` restricts the work to a subset: weight gradients come back as a
    dict keyed by e, and the dXp / dGUp rows of other experts stay zero.
    """
    E = offsets.size - 1
    f = lambda arr: decode(arr, dtype).astype(np.float64)
    M = int(offsets[-1])
    H = W_down.shape[1]
    I = W_down.shape[2]
    dXp = np.zeros((M, H), dtype=np.float64)
    dGUp = np.zeros((M, 2 * I), dtype=np.float64)
    sel = range(E) if experts is None else experts
    dW_down = {}
    dW_gu = {}
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        want_w = e in sel
        if not want_w:
            continue
        if hi == lo:
            if want_w:
                dW_down[e] = np.zeros((H, I))
                dW_gu[e] = np.zeros((2 * I, H))
            continue
        dy = f(DYp[lo:hi])
        g = f(Gp[lo:hi])
        u = f(Up[lo:hi])
        Wd = f(W_down[e])
        Wgu = f(W_gu[e])
        dA = dy @ Wd
        s = sigmoid64(g)
        dG = dA * u * s * (1.0 + g * (1.0 - s))
        dU = dA * g * s
        dGU = np.concatenate([dG, dU], axis=1)
        dGUp[lo:hi] = dGU
        dXp[lo:hi] = dGU @ Wgu
        if want_w:
            dW_down[e] = dy.T @ f(Ap[lo:hi])
            dW_gu[e] = dGU.T @ f(Xp[lo:hi])
    if experts is None:
        dW_down = np.stack([dW_down[e] for e in range(E)])
        dW_gu = np.stack([dW_gu[e] for e in range(E)])
    return dW_down, dW_gu, dXp, dGUp


def expert_backward_rows(rows, offsets, DYp, Gp, Up, W_gu, W_down, dtype: str):
    """dGU_p and dX_p of selected packed rows only (same formulas as expert_backward).

    Each output row depends only on its own packed row and its expert's weights.
    Returns dicts row -> fp64 vector.
    """
    f = lambda arr: decode(arr, dtype).astype(np.float64)
    I = W_down.shape[2]
    rows = np.asarray(sorted(set(int(r) for r in rows)), dtype=np.int64)
    owner = np.searchsorted(np.asarray(offsets), rows, side="right") - 1
    dgu, dxp = {}, {}
    for e in np.unique(owner):
        rs = rows[owner == e]
        dy = f(DYp[rs])
        g = f(Gp[rs])
        u = f(Up[rs])
        dA = dy @ f(W_down[e])
        s = sigmoid64(g)
        dGU = np.concatenate([dA * u * s * (1.0 + g * (1.0 - s)), dA * g * s], axis=1)
        dX = dGU @ f(W_gu[e])
        for i, r in enumerate(rs):
            dgu[int(r)] = dGU[i]
            dxp[int(r)] = dX[i]
    return dgu, dxp


# ----------------------------------------------------------------------------
# a5: back to the token layout
# ----------------------------------------------------------------------------
def unpack_tokens(tokens, dxp_rows, pos, k: int, H: int):
    """dX for selected tokens from a row -> dX_p mapping (same rule as unpack)."""
    pos = np.asarray(pos).reshape(-1, k)
    out = np.zeros((len(tokens), H))
    for i, t in enumerate(tokens):
        for j in range(k):
            r = int(pos[t, j])
            if r >= 0:
                out[i] += dxp_rows[r]
    return out


def unpack(dXp, pos, T: int, k: int):
    """dX[t] = sum over j ascending of dX_p[pos[t*k+j]] for retained pairs; else 0."""
    H = dXp.shape[1]
    dX = np.zeros((T, H), dtype=np.float64)
    pos = np.asarray(pos).reshape(T, k)
    for j in range(k):
        r = pos[:, j]
        keep = r >= 0
        dX[keep] += dXp[r[keep]]
    return dX


def unpack_storage(dXp_stored, pos, T: int, k: int, dtype: str):
    """dX in storage form from dX_p in storage form (R12): per token, acc = +0
    in fp32, then acc = fl(acc + row) for the retained slots j = 0..k-1 in
    order, then one round-to-nearest-even to the storage dtype."""
    rows = decode(np.asarray(dXp_stored), dtype).astype(np.float32)
    pos = np.asarray(pos).reshape(T, k)
    acc = np.zeros((T, rows.shape[1]), dtype=np.float32)
    for j in range(k):
        r = pos[:, j]
        keep = r >= 0
        acc[keep] = acc[keep] + rows[r[keep]]    # float32 + float32: one IEEE rounding
    return encode_rne(acc, dtype)


# ----------------------------------------------------------------------------
# whole path
# ----------------------------------------------------------------------------
def pruned_backward(layer, experts=None):
    """Run a1..a5 on a generated layer.  Returns a dict of every intermediate."""
    s = layer.spec
    dt = s.dtype
    score, st1 = lrm_score(layer.topk_idx, layer.topk_w, layer.dY, layer.a, dt, s.E)
    counts, kept, offsets, perm, pos, st2 = select_quota(layer.topk_idx, score, layer.quota, s.E)
    Xp, DYp, Ap, Gp, Up = pack(perm, layer.topk_w, s.k, layer.x, layer.dY, layer.a, layer.g, layer.u, dt)
    dW_down, dW_gu, dXp, dGUp = expert_backward(Xp, DYp, Ap, Gp, Up, offsets, layer.W_gu,
                                                layer.W_down, dt, experts=experts)
    dX = unpack(dXp, pos, s.T, s.k)
    return dict(score=score, status=st1 | st2, counts=counts, kept=kept, offsets=offsets,
                perm=perm, pos=pos, Xp=Xp, DYp=DYp, Ap=Ap, Gp=Gp, Up=Up,
                dW_down=dW_down, dW_gu=dW_gu, dXp=dXp, dGUp=dGUp, dX=dX)


# ----------------------------------------------------------------------------
# unpruned references (pins only)
# ----------------------------------------------------------------------------
def dense_backward(topk_idx, grad_rows, x, g, u, a, W_gu, W_down):
    """Unpruned expert backward, one pair at a time, in fp64.

    grad_rows[p] is the gradient arriving at expert output y_p (w_p * dY_t,
    already in the precision the caller chose).  Pairs with idx < 0 or idx >= E
    are skipped.  Returns dW_down [E,H,I], dW_gu [E,2I,H], dX [T,H].
    """
    T, k = topk_idx.shape
    E, H, I = W_down.shape
    dW_down = np.zeros((E, H, I))
    dW_gu = np.zeros((E, 2 * I, H))
    dX = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            e = int(topk_idx[t, j])
            if e < 0 or e >= E:
                continue
            p = t * k + j
            gy = grad_rows[p]                                  # dL/dy_p      [H]
            dW_down[e] += np.outer(gy, a[p])                   # dL/dW_down
            da = W_down[e].T @ gy                              # dL/da        [I]
            sg = 1.0 / (1.0 + np.exp(-g[p]))
            silu = g[p] * sg
            dsilu = sg * (1.0 + g[p] * (1.0 - sg))
            dg = da * u[p] * dsilu
            du = da * silu
            dW_gu[e, :I] += np.outer(dg, x[t])
            dW_gu[e, I:] += np.outer(du, x[t])
            dX[t] += W_gu[e, :I].T @ dg + W_gu[e, I:].T @ du
    return dW_down, dW_gu, dX


def forward(topk_idx, topk_w, x, W_gu, W_down):
    """Y_t = sum_j w_tj * W_down[e] (silu(W_gate[e] x_t) * (W_up[e] x_t)), fp64.

    Also returns the saved per-pair g, u, a.
    """
    T, k = topk_idx.shape
    E, H, I = W_down.shape
    Y = np.zeros((T, H))
    g = np.zeros((T * k, I))
    u = np.zeros((T * k, I))
    a = np.zeros((T * k, I))
    for t in range(T):
        for j in range(k):
            e = int(topk_idx[t, j])
            if e < 0 or e >= E:
                continue
            p = t * k + j
            g[p] = W_gu[e, :I] @ x[t]
            u[p] = W_gu[e, I:] @ x[t]
            a[p] = g[p] / (1.0 + np.exp(-g[p])) * u[p]
            Y[t] += topk_w[t, j] * (W_down[e] @ a[p])
    return Y, g, u, a
