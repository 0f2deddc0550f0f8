"""Seeded synthetic MoE layers for the pruned expert backward.

This module only *makes inputs*: router logits, activations, weights, the
upstream gradient, the routing decision and the per-expert quotas, plus the
saved forward activations (g, u, a) that a real forward pass would have kept.
It holds none of the pruned-backward arithmetic (no score, no selection, no
packing, no gradient), so both the CPU oracle and the CUDA path can read the
same bytes from it.

Workload shapes follow the MoE layers named by the LRMoE news pages (Qwen3-30B-A3B
and GLM4.5-106B-A12B, lead paragraph of "LRMoE урезает обратный проход MoE ...")
and the routing / quota rules of the hot-path configurations:

* Routing: softmax(z + b) over E experts, top-k (ties to the lower expert id),
  renormalised k weights.  b_e = log(pop_e), pop_e proportional to (e+1)^-s
  (Zipf skew, expert 0 hottest); no bias for the tiny layer.
* Quotas are integers computed from the routed counts c_e without floats
  (the "quota fixed for the whole layer call" of section "Что делает LRMoE",
  bullet 2; the controller that would choose them is not part of this path).
* bf16 layers store every 16-bit tensor as raw uint16 bit patterns; the fp32
  layer stores float32.

Draw order (numpy default_rng(seed)): z [T,E], x [T,H], W_gu [E,2I,H], W_down
[E,H,I], dY [T,H].  x, W and dY are rounded to the storage dtype (RNE), then
g = x W_gate^T and u = x W_up^T are formed with fp32 accumulation and rounded,
and a = silu(g) * u is formed in fp32 from the rounded g, u and rounded.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

__all__ = ["LayerSpec", "Layer", "CONFIGS", "spec", "make_layer", "quota_from_counts",
           "to_float32", "ALIGN"]

# Feature-dimension granularity the C ABI accepts (16-byte rows for bf16 and fp32).
ALIGN = {"bf16": 8, "f32": 4}


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    name: str
    T: int
    E: int
    k: int
    H: int
    I: int
    dtype: str              # "bf16" or "f32"
    sigma_w: float
    sigma_dy: float
    zipf_s: Optional[float]  # None: no routing bias
    quota: str              # "half_ceil" | "capacity" | "skew" | "keep:<n>/4" | "zero" | "full" | "over"

    @property
    def P(self) -> int:
        return self.T * self.k


CONFIGS: Dict[str, LayerSpec] = {
    # configuration names describe the layer, not a benchmark suite
    "tiny": LayerSpec("tiny", 256, 8, 2, 64, 128, "f32", 0.05, 0.1, None, "half_ceil"),
    "qwen": LayerSpec("qwen", 8192, 128, 8, 2048, 768, "bf16", 0.02, 1e-2, 1.0, "capacity"),
    "glm": LayerSpec("glm", 8192, 128, 8, 4096, 1408, "bf16", 0.02, 1e-2, 1.2, "capacity"),
    "skew": LayerSpec("skew", 32768, 128, 8, 2048, 768, "bf16", 0.02, 1e-2, 1.5, "skew"),
    "sweep100": LayerSpec("sweep100", 16384, 128, 8, 4096, 1408, "bf16", 0.02, 1e-2, 1.2, "keep:4/4"),
    "sweep75": LayerSpec("sweep75", 16384, 128, 8, 4096, 1408, "bf16", 0.02, 1e-2, 1.2, "keep:3/4"),
    "sweep50": LayerSpec("sweep50", 16384, 128, 8, 4096, 1408, "bf16", 0.02, 1e-2, 1.2, "keep:2/4"),
    "sweep25": LayerSpec("sweep25", 16384, 128, 8, 4096, 1408, "bf16", 0.02, 1e-2, 1.2, "keep:1/4"),
}


def spec(name: str, **overrides) -> LayerSpec:
    """A named configuration, optionally with some fields replaced (smaller parity cases)."""
    base = CONFIGS[name]
    if overrides:
        fields = dataclasses.asdict(base)
        fields.update(overrides)
        if "name" not in overrides:
            fields["name"] = base.name + "-" + "-".join(f"{k}{v}" for k, v in sorted(overrides.items()))
        return LayerSpec(**fields)
    return base


def quota_from_counts(counts: np.ndarray, s: LayerSpec) -> np.ndarray:
    """Integer per-expert quotas from routed counts (no floating point)."""
    c = counts.astype(np.int64)
    cap = (s.T * s.k) // s.E
    if s.quota == "half_ceil":
        q = (c + 1) // 2
    elif s.quota == "capacity":
        q = np.minimum(c, cap)
    elif s.quota == "skew":
        q = np.minimum((2 * c + 4) // 5, cap)
    elif s.quota.startswith("keep:"):
        n, d = s.quota[5:].split("/")
        n, d = int(n), int(d)
        q = (n * c + d - 1) // d
    elif s.quota == "zero":
        q = np.zeros_like(c)
    elif s.quota == "full":
        q = c.copy()
    elif s.quota == "over":
        q = c + 7
    else:
        raise ValueError(f"unknown quota rule {s.quota!r}")
    return q.astype(np.int32)


def _round_storage(v: np.ndarray, dtype: str) -> np.ndarray:
    """RNE to the storage dtype via torch's conversion (library routine)."""
    if dtype == "f32":
        return np.ascontiguousarray(v, dtype=np.float32)
    import torch
    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def to_float32(arr: np.ndarray, dtype: str) -> np.ndarray:
    """Storage array -> float32 (bf16 widening is exact)."""
    if dtype == "f32":
        return arr.astype(np.float32, copy=False)
    import torch
    return torch.from_numpy(arr.view(np.int16)).view(torch.bfloat16).float().numpy()


@dataclasses.dataclass
class Layer:
    spec: LayerSpec
    seed: int
    topk_idx: np.ndarray   # int32 [T, k]; <0 = not routed
    topk_w: np.ndarray     # float32 [T, k]
    quota: np.ndarray      # int32 [E]
    x: np.ndarray          # storage [T, H]
    dY: np.ndarray         # storage [T, H]
    W_gu: np.ndarray       # storage [E, 2I, H] (gate rows 0..I-1, up rows I..2I-1)
    W_down: np.ndarray     # storage [E, H, I]
    g: np.ndarray          # storage [P, I]  saved gate pre-activation per pair
    u: np.ndarray          # storage [P, I]  saved up projection per pair
    a: np.ndarray          # storage [P, I]  saved down-projection input silu(g)*u
    counts: np.ndarray     # int64 [E] routed count per expert (input bookkeeping)

    @property
    def dtype(self) -> str:
        return self.spec.dtype


def _route(z: np.ndarray, s: LayerSpec):
    logits = z.astype(np.float64)
    if s.zipf_s is not None:
        e = np.arange(s.E, dtype=np.float64)
        logits = logits - s.zipf_s * np.log(e + 1.0)[None, :]
    logits = logits - logits.max(axis=1, keepdims=True)
    prob = np.exp(logits)
    prob /= prob.sum(axis=1, keepdims=True)
    # ties go to the lower expert id: stable sort of -prob
    order = np.argsort(-prob, axis=1, kind="stable")[:, : s.k]
    w = np.take_along_axis(prob, order, axis=1)
    w = w / w.sum(axis=1, keepdims=True)
    return order.astype(np.int32), w.astype(np.float32)


def _saved_forward(x32, Wgu32, idx, s: LayerSpec, dtype: str):
    """g, u, a for every routed pair, fp32 accumulation, rounded to storage."""
    import torch
    T, k, I = s.T, s.k, s.I
    P = T * k
    g = np.zeros((P, I), dtype=np.float32)
    u = np.zeros((P, I), dtype=np.float32)
    flat = idx.reshape(-1)
    xt = torch.from_numpy(x32)
    for e in range(s.E):
        pairs = np.nonzero(flat == e)[0]
        if pairs.size == 0:
            continue
        rows = xt[torch.from_numpy(pairs // k)]
        gu = rows @ torch.from_numpy(Wgu32[e]).T          # [c_e, 2I] fp32
        g[pairs] = gu[:, :I].numpy()
        u[pairs] = gu[:, I:].numpy()
    g_s = _round_storage(g, dtype)
    u_s = _round_storage(u, dtype)
    g32 = torch.from_numpy(to_float32(g_s, dtype))
    u32 = torch.from_numpy(to_float32(u_s, dtype))
    a32 = (torch.nn.functional.silu(g32) * u32).numpy()
    a_s = _round_storage(a32, dtype)
    return g_s, u_s, a_s


def saved_expert_outputs(layer: "Layer") -> np.ndarray:
    """y_p = W_down[e] a_p for every routed pair (the forward's expert output, which
    it combines as sum_j w_tj y_tj), fp32 accumulation, rounded to storage; zero
    rows for empty and invalid slots.  Computed on demand: [T*k, H] is large."""
    import torch
    s = layer.spec
    k, H = s.k, s.H
    y = np.zeros((s.P, H), dtype=np.float32)
    flat = layer.topk_idx.reshape(-1)
    a32 = torch.from_numpy(to_float32(layer.a, s.dtype))
    for e in range(s.E):
        pairs = np.nonzero(flat == e)[0]
        if pairs.size == 0:
            continue
        Wd = torch.from_numpy(to_float32(layer.W_down[e], s.dtype))   # [H, I]
        y[pairs] = (a32[torch.from_numpy(pairs)] @ Wd.T).numpy()
    return _round_storage(y, s.dtype)


def make_layer(s: LayerSpec | str, seed: int = 0, topk_idx: Optional[np.ndarray] = None,
               quota: Optional[np.ndarray] = None) -> Layer:
    """Draw one synthetic layer.  `topk_idx` / `quota` override routing / quotas (edge cases)."""
    if isinstance(s, str):
        s = CONFIGS[s]
    if s.H % ALIGN[s.dtype] or s.I % ALIGN[s.dtype]:
        raise ValueError("H and I must be multiples of %d for %s" % (ALIGN[s.dtype], s.dtype))
    if s.k > s.E:
        raise ValueError("top-k larger than the number of experts")
    rng = np.random.default_rng(seed)
    T, E, k, H, I = s.T, s.E, s.k, s.H, s.I
    z = rng.standard_normal((T, E), dtype=np.float32)
    x = rng.standard_normal((T, H), dtype=np.float32)
    W_gu = rng.standard_normal((E, 2 * I, H), dtype=np.float32)
    W_gu *= np.float32(s.sigma_w)
    W_down = rng.standard_normal((E, H, I), dtype=np.float32)
    W_down *= np.float32(s.sigma_w)
    dY = rng.standard_normal((T, H), dtype=np.float32)
    dY *= np.float32(s.sigma_dy)

    idx, w = _route(z, s)
    if topk_idx is not None:
        idx = np.ascontiguousarray(topk_idx, dtype=np.int32).reshape(T, k)

    x_s = _round_storage(x, s.dtype)
    dY_s = _round_storage(dY, s.dtype)
    Wgu_s = _round_storage(W_gu, s.dtype)
    Wd_s = _round_storage(W_down, s.dtype)
    del W_gu, W_down
    valid = idx[(idx >= 0) & (idx < E)]
    counts = np.bincount(valid.reshape(-1), minlength=E).astype(np.int64)
    g_s, u_s, a_s = _saved_forward(to_float32(x_s, s.dtype), to_float32(Wgu_s, s.dtype), idx, s, s.dtype)
    if quota is None:
        quota = quota_from_counts(counts, s)
    return Layer(spec=s, seed=seed, topk_idx=idx, topk_w=w, quota=np.asarray(quota, np.int32),
                 x=x_s, dY=dY_s, W_gu=Wgu_s, W_down=Wd_s, g=g_s, u=u_s, a=a_s, counts=counts)

