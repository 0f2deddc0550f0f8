"""Benchmark of the pruned MoE expert backward (LRMoE) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config sweep100] [--impl reference]

A step is one pass of the whole hot path over one synthetic layer: LRM score,
per-expert top-quota selection, compaction, the four grouped GEMMs (SwiGLU
dgrad, dW_down, dW_gate|up, dX_p) and the unpack of dX, issued as the eight
C-ABI calls of liblrmoe.so on one stream.  The metric is retained pairs per
second (plus expert-backward TFLOP/s of the grouped GEMMs), measured with CUDA
events on the launching stream; inputs are resident in HBM and L2 is flushed
between timed steps (a 512 MiB buffer written, then read back), outside the events.

The headline layer is the largest single-GPU configuration: the GLM4.5-106B-A12B-
shaped MoE layer with T = 16384 tokens, E = 128 experts, top-8, H = 4096,
I = 1408, bf16, every routed pair kept (quota = count).  The Qwen3-30B-A3B- and
GLM-shaped T = 8192 layers and the heavy-skew layer are timed after it in the
same run and reported under "other_configs".

N > 1 (torchrun, one process per GPU): every rank runs its own replica of the
layer (the single-GPU path has no exchange step), the timed region is bracketed
by barriers, the max time over ranks is taken, and value = all ranks' retained
pairs / that time ("scaling": "weak").

--impl reference times the CPU oracle (numpy, fp64) on the host cores, one
bounded sample of the same layer per step, and prints the same JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "retained pairs/s + expert-bwd TFLOP/s on 1 B200; % of HBM / bf16 roofline"
UNIT = "retained pairs/s"
DEFAULT_CONFIG = "sweep100"
OTHER_CONFIGS = ("qwen", "glm", "skew")
KERNELS = ("score", "select", "pack", "dgrad_swiglu", "wgrad_down", "wgrad_gu", "dgrad_x", "unpack")
# kernel launches per call: selection is three kernels; each grouped dgrad is a
# two-SM launch for the 256-row tiles plus a one-SM launch for experts' last tiles
KERNEL_LAUNCHES = {"score": 1, "select": 3, "pack": 1, "dgrad_swiglu": 2, "wgrad_down": 1,
                   "wgrad_gu": 1, "dgrad_x": 2, "unpack": 1}
# C-ABI call of each step position (NVTX range names)
CALL_NAMES = ("lrmoe_score", "lrmoe_select_quota", "lrmoe_pack", "lrmoe_grouped_dgrad[swiglu]",
              "lrmoe_grouped_wgrad[down]", "lrmoe_grouped_wgrad[gate|up]",
              "lrmoe_grouped_dgrad[dX]", "lrmoe_unpack")
FUSED_NAMES = ("lrmoe_grouped_dgrad_wgrad[swiglu,down]", "lrmoe_grouped_dgrad_wgrad[dX,gate|up]")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--config", default=DEFAULT_CONFIG)
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--impl", choices=("lrmoe", "reference"), default="lrmoe")
    p.add_argument("--no-cpu-baseline", action="store_true",
                   help="skip timing the CPU oracle (profiling runs)")
    p.add_argument("--sweep", action="store_true",
                   help="quota sweep (keep 1, 3/4, 1/2, 1/4) on the GLM-shaped T=16384 layer")
    p.add_argument("--no-extras", action="store_true",
                   help="time only the step (profiling runs): no controller, fused-GEMM, "
                        "saved-norm, routing-gradient, redistribution or end-to-end blocks")
    p.add_argument("--cpu-budget", type=float, default=20.0,
                   help="seconds of host time for the bounded oracle sample (cpu_baseline)")
    p.add_argument("--override", default="",
                   help="layer fields to replace, e.g. T=4096,E=64 (smaller profiling cases)")
    return p.parse_args(argv)


def layer_spec(args):
    from pruned_expert_backward_lrmoe_b200 import inputs
    over = {}
    for item in filter(None, args.override.split(",")):
        key, val = item.split("=")
        over[key] = val if key in ("quota", "dtype", "name") else int(val)
    return inputs.spec(args.config, **over)


# ---------------------------------------------------------------------------
# algorithmic bytes and flops per launch (per kernel), from the layer's sizes
# ---------------------------------------------------------------------------
def algorithmic(T, k, E, H, I, M, b):
    """Bytes each step must move at minimum, and the grouped-GEMM flops."""
    P = T * k
    by = {
        "score": T * H * b + P * I * b + 8 * P + 4 * P,
        "select": 4 * P + 4 * P + 4 * E + 12 * E + 4 * M + 4 * P,
        # bf16 path: X_p, DY_p, A_p (g, u are read in place at row perm[r]);
        # fp32: X_p, DY_p, A_p, G_p, U_p
        "pack": 2 * M * (2 * H + (I if b == 2 else 3 * I)) * b + 8 * M,
        "dgrad_swiglu": M * H * b + E * H * I * b + 2 * M * I * b + 2 * M * I * b,
        "wgrad_down": M * H * b + M * I * b + E * H * I * 4,
        "wgrad_gu": 2 * M * I * b + M * H * b + E * 2 * I * H * 4,
        "dgrad_x": 2 * M * I * b + E * 2 * I * H * b + M * H * b,
        "unpack": M * H * b + 4 * P + T * H * b,
    }
    fl = {"dgrad_swiglu": 2 * M * H * I, "wgrad_down": 2 * M * H * I, "wgrad_gu": 4 * M * I * H,
          "dgrad_x": 4 * M * I * H}
    # fused launches: the shared gradient rows (DY_p, dGU_p) count once
    by["dgrad_swiglu+wgrad_down"] = by["dgrad_swiglu"] + by["wgrad_down"] - M * H * b
    by["dgrad_x+wgrad_gu"] = by["dgrad_x"] + by["wgrad_gu"] - 2 * M * I * b
    fl["dgrad_swiglu+wgrad_down"] = fl["dgrad_swiglu"] + fl["wgrad_down"]
    fl["dgrad_x+wgrad_gu"] = fl["dgrad_x"] + fl["wgrad_gu"]
    return by, fl


def step_gemms(fl):
    """The grouped-GEMM entries of KERNELS (the step's launches)."""
    return [n for n in KERNELS if n in fl]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# the sources that define each kernel whose DRAM traffic is recorded
_GEMM_SOURCES = ("gemm_tc.cu", "gemm_pair.cu", "gemm_common.cuh", "common.cuh", "grouped.cuh",
                 "launch.h")
KERNEL_SOURCES = {
    "score": ("score.cu", "rowreduce.cuh", "common.cuh"),
    "select": ("select.cu", "grouped.cuh", "common.cuh"),
    "pack": ("pack.cu", "common.cuh"),
    "unpack": ("pack.cu", "common.cuh"),
    "dgrad_swiglu": _GEMM_SOURCES, "wgrad_down": _GEMM_SOURCES,
    "wgrad_gu": _GEMM_SOURCES, "dgrad_x": _GEMM_SOURCES,
}
GEMM_SOURCES = _GEMM_SOURCES


def _code_only(text: str) -> str:
    """C++/CUDA source without comments and with whitespace runs collapsed, so that an
    edit of comments alone does not count as a change of the kernel."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_sha1(kernel: str = "wgrad_gu") -> str:
    """sha1 over the code (comments dropped) of the source files that define `kernel`."""
    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "pruned_expert_backward_lrmoe_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode())
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()


def recorded_traffic(kernel: str, config: str, algorithmic_bytes: float | None = None):
    """DRAM bytes per launch of `kernel` on layer `config` from a committed ncu summary.

    profiles/traffic.json maps "<kernel>@<layer>" to {"bytes": B, "source_sha1": S}
    (captured on that layer), or to {"bytes": B, "algorithmic_bytes": A,
    "scale_to": [layers], ...} for a capture on a smaller case of the same kernel,
    which is scaled to a full launch of each listed layer as B / A x that launch's
    algorithmic bytes.  Returns (bytes, how) or (None, reason); a figure is dropped
    when the kernel's own sources changed since the capture.
    """
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            table = json.load(f)
    except (OSError, ValueError):
        return None, "no profiles/traffic.json"
    sha = kernel_source_sha1(kernel)
    ent = table.get(f"{kernel}@{config}")
    if ent:
        if ent.get("source_sha1") != sha:
            return None, "kernel changed since the capture"
        return ent.get("bytes"), "ncu capture of this launch"
    for key, ent in table.items():
        if key.split("@")[0] != kernel or config not in ent.get("scale_to", ()):
            continue
        if ent.get("source_sha1") != sha:
            return None, "kernel changed since the capture"
        if algorithmic_bytes is None or not ent.get("algorithmic_bytes"):
            return None, "no algorithmic bytes to scale by"
        ratio = ent["bytes"] / ent["algorithmic_bytes"]
        return ratio * algorithmic_bytes, f"scaled from the ncu capture {key} (traffic/algorithmic {ratio:.3f})"
    return None, "not captured"


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, sampled from a thread)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {  # NVML clocks-event reason bits
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: clocks are reported as unknown
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
                self.reasons |= int(get(self._h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        reasons = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}; launch N>1 with torchrun")
    if world == 1:
        return 0, 1, 0, None
    import datetime

    import torch
    import torch.distributed as dist
    rank, local = int(os.environ["RANK"]), int(os.environ.get("LOCAL_RANK", "0"))
    backend = "nccl" if torch.cuda.is_available() else "gloo"
    if backend == "nccl":
        torch.cuda.set_device(local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world, local, dist


def max_over_ranks(value: float, dist) -> float:
    if dist is None:
        return value
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, dist) -> float:
    if dist is None:
        return value
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(dist):
    if dist is not None:
        dist.barrier()


# ---------------------------------------------------------------------------
# CPU oracle timings
# ---------------------------------------------------------------------------
def oracle_full_pass(layer):
    """One pass of the oracle over the whole layer; returns (seconds, retained pairs)."""
    from oracle import lrmoe_oracle as O
    t0 = time.perf_counter()
    r = O.pruned_backward(layer)
    return time.perf_counter() - t0, int(r["offsets"][-1])


def oracle_expert_sample(layer, experts):
    """The oracle on the pairs of a few experts, as a standalone mini layer per expert.

    Each expert's routed pairs become a layer with k = 1 and one expert; the
    oracle runs score, selection, compaction, backward and unpack on it.
    Returns (seconds, retained pairs).
    """
    from oracle import lrmoe_oracle as O
    s = layer.spec
    flat = layer.topk_idx.reshape(-1)
    done = 0
    t0 = time.perf_counter()
    for e in experts:
        pairs = np.nonzero(flat == e)[0]
        if pairs.size == 0:
            continue
        tok = pairs // s.k
        idx = np.zeros((pairs.size, 1), np.int32)
        w = layer.topk_w.reshape(-1)[pairs].reshape(-1, 1)
        score, _ = O.lrm_score(idx, w, layer.dY[tok], layer.a[pairs], s.dtype, 1)
        _, _, off, perm, pos, _ = O.select_quota(idx, score, layer.quota[e:e + 1], 1)
        Xp, DYp, Ap, Gp, Up = O.pack(perm, w, 1, layer.x[tok], layer.dY[tok], layer.a[pairs],
                                     layer.g[pairs], layer.u[pairs], s.dtype)
        _, _, dXp, _ = O.expert_backward(Xp, DYp, Ap, Gp, Up, off, layer.W_gu[e:e + 1],
                                         layer.W_down[e:e + 1], s.dtype)
        O.unpack(dXp, pos, pairs.size, 1)
        done += int(off[-1])
    return time.perf_counter() - t0, done


def host_cores() -> int:
    """Threads the oracle's arithmetic runs on: numpy's BLAS pool (its matmuls are
    the oracle's heavy steps), else torch's CPU thread count."""
    try:
        import threadpoolctl
        for pool in threadpoolctl.threadpool_info():
            if pool.get("user_api") == "blas":
                return int(pool["num_threads"])
    except Exception:
        pass
    try:
        import torch
        return int(torch.get_num_threads())
    except Exception:
        return os.cpu_count() or 1


def oracle_bounded_sample(layer, budget_s: float = 20.0):
    """The oracle on a bounded sample of the layer: whole experts as standalone k = 1
    layers (score, selection, compaction, fp64 backward, unpack), taken in the
    order e = E/2, E/2 + 1, ... (wrapping), until about `budget_s` seconds of host
    time are spent.  Returns (seconds, retained pairs, experts done)."""
    E = layer.spec.E
    tot_s, tot_m, done = 0.0, 0, []
    for i in range(E):
        if tot_s >= budget_s:
            break
        e = (E // 2 + i) % E
        dt_, m = oracle_expert_sample(layer, [e])
        tot_s += dt_
        tot_m += m
        done.append(e)
    return tot_s, tot_m, done


def host_cpu() -> dict:
    """nproc and the CPU model name, reported beside every oracle timing."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count() or 1, "cpu_model": model}


def run_reference(args):
    """The oracle on the host cores, one bounded expert sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from pruned_expert_backward_lrmoe_b200 import inputs
    layer = inputs.make_layer(layer_spec(args), seed=args.seed)
    s = layer.spec
    E = s.E
    # size the per-step sample so that warmup + steps end within ~3 minutes
    t_one, _ = oracle_expert_sample(layer, [0])
    per_step_budget = 150.0 / max(1, args.steps + args.warmup)
    group = int(max(1, min(E, per_step_budget / max(t_one, 1e-3))))
    nxt = 0
    for _ in range(args.warmup):
        oracle_expert_sample(layer, [(nxt + i) % E for i in range(group)])
        nxt = (nxt + group) % E
    tot_s, tot_m = 0.0, 0
    for _ in range(args.steps):
        dt_, m = oracle_expert_sample(layer, [(nxt + i) % E for i in range(group)])
        nxt = (nxt + group) % E
        tot_s += dt_
        tot_m += m
    value = tot_m / tot_s if tot_s > 0 else 0.0
    cores = host_cores()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot_s / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(s, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{group} expert(s) per step as standalone k=1 layers "
                                   f"(score, selection, compaction, fp64 backward, unpack)",
                         **host_cpu()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


LAYER_SHAPES = {"tiny": "tiny fp32 MoE layer", "qwen": "Qwen3-30B-A3B-shaped MoE layer",
                "glm": "GLM4.5-106B-A12B-shaped MoE layer",
                "skew": "heavy-skew (Zipf 1.5) Qwen3-30B-A3B-shaped MoE layer",
                "sweep": "GLM4.5-106B-A12B-shaped MoE layer"}


def quota_rule(q: str) -> str:
    if q.startswith("keep:"):
        n, d = q[5:].split("/")
        return "every routed pair kept (quota = count)" if n == d else \
            f"keep {n}/{d} of each expert's pairs (quota = ceil({n}*count/{d}))"
    return {"capacity": "quota = min(count, T*k/E)",
            "skew": "quota = min(ceil(0.4*count), T*k/E)",
            "half_ceil": "quota = ceil(count/2)"}.get(q, f"quota rule '{q}'")


def config_block(s, n_gpus):
    base = next((v for k_, v in LAYER_SHAPES.items() if s.name.startswith(k_)), "MoE layer")
    return {"workload": f"{base} ({s.name}), pruned expert backward: T={s.T} E={s.E} top-{s.k} "
                        f"H={s.H} I={s.I} {s.dtype}, {quota_rule(s.quota)}",
            "layer": s.name, "quota": s.quota,
            "T": s.T, "E": s.E, "k": s.k, "H": s.H, "I": s.I, "global_batch": s.T * n_gpus,
            "parallelism": f"replicas x{n_gpus}" if n_gpus > 1 else "single GPU",
            "l2": "flushed between timed steps (512 MiB written, then read back); inputs also exceed L2"}


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------
def make_runner(layer, dev):
    """Device copies of a layer, output buffers, an L2 flush and the step (eight C-ABI calls)."""
    import torch

    from pruned_expert_backward_lrmoe_b200 import lrmoe as L

    s = layer.spec
    tdt = torch.bfloat16 if s.dtype == "bf16" else torch.float32
    nvtx = torch.cuda.nvtx

    def storage(arr):
        if s.dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(arr))

    host = {"topk_idx": torch.from_numpy(layer.topk_idx), "topk_w": torch.from_numpy(layer.topk_w),
            "quota": torch.from_numpy(layer.quota), "x": storage(layer.x), "dY": storage(layer.dY),
            "g": storage(layer.g), "u": storage(layer.u), "a": storage(layer.a)}
    weights = {"W_gu": storage(layer.W_gu).to(dev), "W_down": storage(layer.W_down).to(dev)}
    inp = {k_: v.to(dev) for k_, v in host.items()}
    inp.update(weights)
    out = L.alloc_buffers(s.T, s.k, s.E, s.H, s.I, tdt, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(128 << 20, dtype=torch.float32, device=dev)  # 512 MiB > 126 MB L2

    def flush_l2():
        # write the buffer (evicts everything), then read it back so that the
        # dirty lines are written out here rather than by the next timed kernel
        flush.zero_()
        flush.sum()
    st = out["status"]

    def step(ev=None, a_sqnorm=None, fused=False, wgrad_gather=False, waits=None, src=None):
        """One pass of the path; with a_sqnorm (||a_p||^2 saved by the forward) the
        score reads dY and the saved norms instead of a; `src` replaces the device
        inputs (a second set, for uploads that overlap the previous step)."""
        inp_ = inp if src is None else src
        gather = s.dtype == "bf16" and not fused   # the path's g, u handling
        score_call = (
            (lambda: L.lrmoe_score(inp_["topk_idx"], inp_["topk_w"], inp_["dY"], inp_["a"], s.E,
                                   out["score"], st, stream)) if a_sqnorm is None else
            (lambda: L.lrmoe_score_from_norms(inp_["topk_idx"], inp_["topk_w"], inp_["dY"], a_sqnorm,
                                              s.E, out["score"], st, stream)))
        head = (
            score_call,
            lambda: L.lrmoe_select_quota(inp_["topk_idx"], out["score"], inp_["quota"], out["counts"],
                                         out["kept"], out["offsets"], out["perm"], out["pos"],
                                         out["workspace"], st, stream),
            # bf16: g, u are read in place at row perm[r] (and, with wgrad_gather, a, x)
            (lambda: L.lrmoe_pack(out["perm"], out["offsets"], inp_["topk_w"], None, inp_["dY"],
                                  None, None, None, None, out["DYp"], None, None, None, st,
                                  stream, I=s.I)) if gather and wgrad_gather else
            (lambda: L.lrmoe_pack(out["perm"], out["offsets"], inp_["topk_w"], inp_["x"], inp_["dY"],
                                  inp_["a"], None, None, out["Xp"], out["DYp"], out["Ap"], None,
                                  None, st, stream)) if gather else
            (lambda: L.lrmoe_pack(out["perm"], out["offsets"], inp_["topk_w"], inp_["x"], inp_["dY"],
                                  inp_["a"], inp_["g"], inp_["u"], out["Xp"], out["DYp"], out["Ap"],
                                  out["Gp"], out["Up"], st, stream)),
        )
        if not fused:  # the four grouped GEMMs as separate launches
            gemms = (
                (lambda: L.lrmoe_grouped_dgrad_swiglu_gather(
                    out["DYp"], inp_["W_down"], out["offsets"], out["perm"], inp_["g"], inp_["u"],
                    out["dGUp"], status=st, stream=stream)) if gather else
                (lambda: L.lrmoe_grouped_dgrad(out["DYp"], inp_["W_down"], out["offsets"],
                                               L.LRMOE_EPI_SWIGLU_BWD, out["dGUp"], Gp=out["Gp"],
                                               Up=out["Up"], status=st, stream=stream)),
                (lambda: L.lrmoe_grouped_wgrad_gather(
                    out["DYp"], out["perm"], inp_["a"], 1, s.P, out["offsets"], out["dW_down"],
                    status=st, stream=stream)) if gather and wgrad_gather else
                (lambda: L.lrmoe_grouped_wgrad(out["DYp"], out["Ap"], out["offsets"],
                                               out["dW_down"], status=st, stream=stream)),
                (lambda: L.lrmoe_grouped_wgrad_gather(
                    out["dGUp"], out["perm"], inp_["x"], s.k, s.P, out["offsets"], out["dW_gu"],
                    status=st, stream=stream)) if gather and wgrad_gather else
                (lambda: L.lrmoe_grouped_wgrad(out["dGUp"], out["Xp"], out["offsets"],
                                               out["dW_gu"], status=st, stream=stream)),
                lambda: L.lrmoe_grouped_dgrad(out["dGUp"], inp_["W_gu"], out["offsets"],
                                              L.LRMOE_EPI_STORE, out["dXp"], status=st,
                                              stream=stream),
            )
        else:  # each dgrad with the wgrad over the same gradient rows in one launch
            gemms = (
                lambda: L.lrmoe_grouped_dgrad_wgrad(
                    out["DYp"], inp_["W_down"], out["offsets"], L.LRMOE_EPI_SWIGLU_BWD,
                    out["dGUp"], out["Ap"], out["dW_down"], Gp=out["Gp"], Up=out["Up"],
                    status=st, stream=stream),
                lambda: L.lrmoe_grouped_dgrad_wgrad(
                    out["dGUp"], inp_["W_gu"], out["offsets"], L.LRMOE_EPI_STORE, out["dXp"],
                    out["Xp"], out["dW_gu"], status=st, stream=stream),
            )
        calls = head + gemms + (
            lambda: L.lrmoe_unpack(out["dXp"], out["pos"], s.T, s.k, out["dX"], st, stream),)
        names = CALL_NAMES if not fused else CALL_NAMES[:3] + FUSED_NAMES + CALL_NAMES[-1:]
        for i, c in enumerate(calls):
            if waits and i in waits:
                for ev_ in waits[i]:
                    stream.wait_event(ev_)
            if ev is not None:
                ev[i].record(stream)
            nvtx.range_push(names[i])   # one NVTX range per C-ABI call
            c()
            nvtx.range_pop()
        if ev is not None:
            ev[len(calls)].record(stream)

    return host, inp, out, stream, flush_l2, step


def roofline_of(kname, ms, by, fl, peaks, peak_src, layer_name):
    """Roofline entry of one kernel: the bound (tensor when its flops per algorithmic
    byte exceed the ridge of the peaks, else HBM), achieved = algorithmic flops or
    bytes per launch / measured launch time, and the recorded DRAM traffic."""
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    tf = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    ridge = tf * 1e12 / (hbm * 1e9)
    flops, nbytes = fl.get(kname, 0), by[kname]
    if flops and flops / nbytes > ridge:
        ach = flops / (ms * 1e-3) / 1e12
        bound, peak, unit, src = "tensor", tf, "TFLOP/s", f"{peak_src} bf16_tflops_sustained"
    else:
        ach = nbytes / (ms * 1e-3) / 1e9
        bound, peak, unit, src = "hbm", hbm, "GB/s", f"{peak_src} hbm_gbs"
    traffic, how = recorded_traffic(kname, layer_name, nbytes)
    return {"kernel": kname, "bound": bound, "achieved": ach, "peak": peak, "unit": unit,
            "frac": ach / peak, "traffic": traffic, "traffic_source": how,
            "peak_source": src, "algorithmic_bytes": nbytes, "algorithmic_flops": flops,
            "flop_per_byte": flops / nbytes, "ridge_flop_per_byte": ridge, "ms": ms}


def measure_layer(layer, dev, steps, warmup, dist, peaks, peak_src, breakdown_steps=None):
    """Time K steps of the path on one layer (L2 flushed between steps), then a
    second pass with events between the calls for per-kernel durations."""
    import torch

    s = layer.spec
    b = 2 if s.dtype == "bf16" else 4
    runner = make_runner(layer, dev)
    host, inp, out, stream, flush_l2, step = runner
    st = out["status"]
    st.zero_()
    for _ in range(max(1, warmup)):
        step()
    torch.cuda.synchronize(dev)
    if int(st.item()) != 0:
        raise SystemExit(f"device status {int(st.item())} after warm-up ({s.name})")
    M = int(out["offsets"][-1].item())
    counts = out["kept"].cpu().numpy()

    # Headline: K steps with events only around each step (events between the
    # kernels would stop each kernel's launch from overlapping its predecessor's
    # tail).  Then a second timed pass with events between the eight calls gives
    # the per-kernel durations used for the breakdown and the roofline.
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    n_bd = breakdown_steps or max(3, min(steps, 50))
    evs_bd = [[torch.cuda.Event(enable_timing=True) for _ in range(len(KERNELS) + 1)]
              for _ in range(n_bd)]
    with ClockSampler(dev.index or 0) as clk:
        barrier(dist)
        torch.cuda.synchronize(dev)
        for i in range(steps):
            flush_l2()
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
        barrier(dist)
        for i in range(n_bd):
            flush_l2()
            step(evs_bd[i])
        torch.cuda.synchronize(dev)
        barrier(dist)
    if int(st.item()) != 0:
        raise SystemExit(f"device status {int(st.item())} after the timed steps ({s.name})")
    per_kernel = {kname: [] for kname in KERNELS}
    for ev in evs_bd:
        for j, kname in enumerate(KERNELS):
            per_kernel[kname].append(ev[j].elapsed_time(ev[j + 1]))
    step_ms = [a_.elapsed_time(b_) for a_, b_ in evs]
    mean_step = statistics.fmean(step_ms)
    mean_step_max = max_over_ranks(mean_step, dist)
    M_all = sum_over_ranks(float(M), dist)
    kern_ms = {kname: statistics.fmean(v) for kname, v in per_kernel.items()}
    by, fl = algorithmic(s.T, s.k, s.E, s.H, s.I, M, b)
    gemm_ms = sum(kern_ms[n] for n in step_gemms(fl))
    gemm_flops = sum(fl[n] for n in step_gemms(fl))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    tf_peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    breakdown = {}
    for kname in KERNELS:
        r = roofline_of(kname, kern_ms[kname], by, fl, peaks, peak_src, s.name)
        e = {"ms": kern_ms[kname], "bound": r["bound"], "frac": r["frac"],
             "GB/s": by[kname] / (kern_ms[kname] * 1e-3) / 1e9}
        e["hbm_frac"] = e["GB/s"] / hbm_peak
        if kname in fl:
            e["TFLOP/s"] = fl[kname] / (kern_ms[kname] * 1e-3) / 1e12
            e["tensor_frac"] = e["TFLOP/s"] / tf_peak
        if r["traffic"] is not None:
            e["traffic"] = r["traffic"]
        breakdown[kname] = e
    dominant = max(kern_ms, key=kern_ms.get)
    return {
        "runner": runner, "M": M, "M_all": M_all, "counts": counts,
        "ms_per_step": mean_step_max, "value": M_all / (mean_step_max * 1e-3),
        "kern_ms": kern_ms, "breakdown": breakdown, "breakdown_steps": n_bd,
        "breakdown_step_ms": sum(kern_ms.values()),
        "gemm_ms": gemm_ms, "expert_bwd_tflops": gemm_flops / (gemm_ms * 1e-3) / 1e12,
        "roofline": roofline_of(dominant, kern_ms[dominant], by, fl, peaks, peak_src, s.name),
        "clocks": clk.summary(), "by": by, "fl": fl,
    }


def run_extras(layer, res, dev, args, dist, peaks):
    """Blocks timed on the headline layer after the step: quota controller, score from
    saved norms, fused and gathering GEMM variants, routing-weight gradient,
    redistribution split, and the end-to-end number through host buffers."""
    import torch

    from pruned_expert_backward_lrmoe_b200 import lrmoe as L

    s = layer.spec
    b = 2 if s.dtype == "bf16" else 4
    tdt = torch.bfloat16 if s.dtype == "bf16" else torch.float32
    host, inp, out, stream, flush_l2, step = res["runner"]
    st = out["status"]
    M, M_all, n_bd = res["M"], res["M_all"], res["breakdown_steps"]
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    x = {}

    def timed(fn, n=20, warm=3, flush=True):
        evp = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for i in range(n + warm):
            if flush:
                flush_l2()
            if i >= warm:
                evp[i - warm][0].record(stream)
            fn()
            if i >= warm:
                evp[i - warm][1].record(stream)
        torch.cuda.synchronize(dev)
        return statistics.fmean(a_.elapsed_time(b_) for a_, b_ in evp)

    # ---------------- quota controller (runs before the backward; not in the step) ----------------
    q_dev = torch.empty(s.E, dtype=torch.int32, device=dev)
    c_dev = torch.empty(s.E, dtype=torch.int32, device=dev)
    cap = (s.T * s.k) // s.E
    x["quota_controller_us"] = 1e3 * timed(
        lambda: L.lrmoe_quota_controller(inp["topk_idx"], s.E, cap, -1, q_dev, c_dev, st, stream),
        flush=False)
    x["quota_controller_equals_capacity_rule"] = (
        bool(torch.equal(q_dev, inp["quota"])) if s.quota == "capacity" else None)

    # ---------------- score from forward-saved ||a_p||^2 ----------------
    # The forward can save ||a_p||^2 when it writes a; the backward's score then
    # reads dY and 4 bytes per pair.  Timed per call after an L2 flush, and as
    # whole steps with that score in place of the full one.
    a2d = inp["a"].view(s.P, s.I)
    na = torch.empty(s.P, dtype=torch.float32, device=dev)
    L.lrmoe_row_sqnorm(a2d, na, stream)
    sn_us = {
        "row_sqnorm": 1e3 * timed(lambda: L.lrmoe_row_sqnorm(a2d, na, stream)),
        "score_from_norms": 1e3 * timed(lambda: L.lrmoe_score_from_norms(
            inp["topk_idx"], inp["topk_w"], inp["dY"], na, s.E, out["score"], st, stream)),
        "score": 1e3 * timed(lambda: L.lrmoe_score(inp["topk_idx"], inp["topk_w"], inp["dY"],
                                                   inp["a"], s.E, out["score"], st, stream)),
    }

    def step_ms(**kw):
        evp = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n_bd)]
        for i in range(n_bd):
            flush_l2()
            evp[i][0].record(stream)
            step(**kw)
            evp[i][1].record(stream)
        torch.cuda.synchronize(dev)
        return max_over_ranks(statistics.fmean(a_.elapsed_time(b_) for a_, b_ in evp), dist)

    sn_step = step_ms(a_sqnorm=na)
    sn_bytes = s.T * s.H * b + 16 * s.P          # dY, idx, w, saved norm, score
    x["saved_norms"] = {
        "row_sqnorm_us": sn_us["row_sqnorm"], "score_from_norms_us": sn_us["score_from_norms"],
        "score_us": sn_us["score"],
        "score_from_norms_GB/s": sn_bytes / (sn_us["score_from_norms"] * 1e-6) / 1e9,
        "score_from_norms_hbm_frac": sn_bytes / (sn_us["score_from_norms"] * 1e-6) / 1e9 / hbm_peak,
        "step_ms": sn_step, "value": M_all / (sn_step * 1e-3), "unit": UNIT, "steps": n_bd,
    }
    # the same steps with each dgrad and its wgrad fused into one launch, and with
    # the wgrads gathering a, x in place (only DY_p packed)
    x["fused_gemm_step_ms"] = step_ms(fused=True)
    x["gathered_wgrad_step_ms"] = step_ms(wgrad_gather=True)
    if int(st.item()) != 0:
        raise SystemExit(f"device status {int(st.item())} after the variant steps")

    # ---------------- routing-weight gradient from saved expert outputs ----------------
    # y_p = W_down[e] a_p is what the forward saves; it is generated here with torch
    # (input generation, not part of the path), then dw = <dY_t, y_p> is timed for
    # the retained pairs (pos from the selection) and for every routed pair.
    y_dev = torch.empty(s.P, s.H, dtype=tdt, device=dev)
    flat_idx = inp["topk_idx"].view(-1)
    for e in range(s.E):
        sel = (flat_idx == e).nonzero().squeeze(1)
        if sel.numel():
            y_dev[sel] = a2d[sel] @ inp["W_down"][e].T
    dw = torch.empty(s.P, dtype=torch.float32, device=dev)
    router = {}
    for mode, pos_arg, nbytes in (
            ("retained", out["pos"], M * s.H * b + s.T * s.H * b + 12 * s.P),
            ("all", None, s.P * s.H * b + s.T * s.H * b + 8 * s.P)):
        us = 1e3 * timed(lambda: L.lrmoe_router_grad(inp["topk_idx"], inp["dY"], y_dev, s.E, dw,
                                                     pos=pos_arg, status=st, stream=stream))
        gbs = nbytes / (us * 1e-6) / 1e9
        router[mode] = {"us": us, "GB/s": gbs, "hbm_frac": gbs / hbm_peak,
                        "algorithmic_bytes": nbytes}
    x["router_grad"] = router
    del y_dev
    if int(st.item()) != 0:
        raise SystemExit(f"device status {int(st.item())} after the router gradient")

    # ---------------- redistribution over expert copies (one rank's view) ----------------
    # An 8-GPU copy map: expert e at home on GPU e % 8, the 16 most loaded experts with
    # a second copy three GPUs on.  The host planner's time and peak against an even
    # split and against home-only placement; then this rank's rows cut by the plan.
    G_plan = 8
    m_np = out["kept"].cpu().numpy().astype(np.int64)
    adm = np.zeros((s.E, G_plan), bool)
    adm[np.arange(s.E), np.arange(s.E) % G_plan] = True
    hot = np.argsort(-m_np, kind="stable")[:16]
    adm[hot, (hot + 3) % G_plan] = True
    t0 = time.perf_counter()
    plan, peak = L.lrmoe_redistribute(m_np, adm)
    planner_us = (time.perf_counter() - t0) * 1e6
    home = np.bincount(np.arange(s.E) % G_plan, weights=m_np, minlength=G_plan)
    plan_dev = torch.from_numpy(plan.astype(np.int32)).to(dev)
    pd = torch.empty(s.P, dtype=torch.int32, device=dev)
    do = torch.empty(G_plan + 1, dtype=torch.int32, device=dev)
    deo = torch.empty(G_plan, s.E + 1, dtype=torch.int32, device=dev)
    split_ms = timed(lambda: L.lrmoe_split_by_destination(out["perm"], out["offsets"], plan_dev,
                                                          pd, do, deo, status=st, stream=stream))
    x["redistribution"] = {
        "gpus_in_plan": G_plan, "copies": int(adm.sum()), "planner_us": planner_us,
        "peak": int(peak), "even_split": int(-(-int(m_np.sum()) // G_plan)),
        "home_only_peak": int(home.max()), "split_us": 1e3 * split_ms,
    }
    if int(st.item()) != 0:
        raise SystemExit(f"device status {int(st.item())} after the destination split")

    # ---------------- the redistributed backward at world size 1 ----------------
    # exchange.redistributed_backward on this layer with one rank: the same GEMMs as
    # the step plus the exchange bookkeeping (split by receiver, wide exchange rows,
    # grouping of the received rows, their split, the return gathers) and its two
    # host synchronisations; the all-to-alls are local copies at this size.
    from pruned_expert_backward_lrmoe_b200 import exchange as X
    ones = np.ones((s.E, 1), bool)
    ex_st = {}
    ex_ms = timed(lambda: ex_st.update(X.redistributed_backward(inp, ones)), n=5, warm=2)
    x["exchange_world1"] = {"ms": ex_ms, "step_ms": res["ms_per_step"],
                            "value": M_all / (ex_ms * 1e-3),
                            "unit": UNIT, "status": int(ex_st["status"].item())}
    del ex_st
    torch.cuda.empty_cache()
    return x


def run_e2e(layer, res, dev, args, dist):
    """The same metric end to end: every step uploads its inputs from pinned host
    memory, runs the path and reads dX and the status word back, all inside the timed
    region.  Steps are pipelined over two sets of device input buffers: the uploads of
    step j+1 (two copy streams, in the order the path consumes them) run while step j
    computes, and step j's dX goes back on a third stream.  The timed region spans the
    whole run, from the first upload to the last read-back; the value is the retained
    pairs of all steps over that time."""
    import torch

    s = layer.spec
    tdt = torch.bfloat16 if s.dtype == "bf16" else torch.float32
    host, inp, out, stream, flush_l2, step = res["runner"]
    pin = {k_: v.pin_memory() for k_, v in host.items()}
    sets = (inp, dict(inp, **{k_: torch.empty_like(inp[k_]) for k_ in pin}))
    dX_host = [torch.empty(s.T, s.H, dtype=tdt).pin_memory() for _ in range(2)]
    st_host = [torch.zeros(1, dtype=torch.int32).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pin.values())
    d2h = dX_host[0].numel() * dX_host[0].element_size() + 4
    n_e2e = max(3, min(args.steps, 50))
    # The compute stream waits only where it needs each group (score and select:
    # routing, dY, a; pack: x; the SwiGLU dgrad: g, u), and its unpack (the last call,
    # which writes dX) for the read-back of the previous step's dX.  Each group's
    # tensors are split over two copy streams (two DMA queues in flight at once).
    copy_streams = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
    back = torch.cuda.Stream(dev)
    groups = (("topk_idx", "topk_w", "quota", "dY", "a"), ("x",), ("g", "u"))
    need_at = (0, 2, 3)   # step call index before which each group must have landed
    unpack_at = len(CALL_NAMES) - 1

    def upload(j, after):
        """Step j's uploads into input set j % 2, once the event `after` has passed."""
        dst = sets[j % 2]
        for cs in copy_streams:
            cs.wait_event(after)
        landed = []
        for grp in groups:
            evs_ = []
            for c, cs in enumerate(copy_streams):
                with torch.cuda.stream(cs):
                    for k_ in grp:
                        half = pin[k_].shape[0] // 2
                        rows = slice(0, half) if c == 0 else slice(half, None)
                        if pin[k_][rows].numel():
                            dst[k_][rows].copy_(pin[k_][rows], non_blocking=True)
                    ev_ = torch.cuda.Event()
                    ev_.record(cs)
                    evs_.append(ev_)
            landed.append(evs_)
        return landed

    def run(n):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        done, read, landed = [None] * n, [None] * n, {0: upload(0, t0)}
        for j in range(n):
            if j + 1 < n:   # set (j+1) % 2 was last read by step j-1
                landed[j + 1] = upload(j + 1, done[j - 1] if j >= 1 else t0)
            flush_l2()
            waits = dict(zip(need_at, landed.pop(j)))
            if j >= 1:
                waits.setdefault(unpack_at, []).append(read[j - 1])
            step(waits=waits, src=sets[j % 2])
            done[j] = torch.cuda.Event()
            done[j].record(stream)
            back.wait_event(done[j])
            with torch.cuda.stream(back):
                dX_host[j % 2].copy_(out["dX"], non_blocking=True)
                st_host[j % 2].copy_(out["status"], non_blocking=True)
                read[j] = torch.cuda.Event()
                read[j].record(back)
        stream.wait_event(read[n - 1])
        t1.record(stream)
        torch.cuda.synchronize(dev)
        return t0.elapsed_time(t1)

    run(2)   # warm-up
    e2e_ms = max_over_ranks(run(n_e2e) / n_e2e, dist)
    bad = [int(h.item()) for h in st_host if int(h.item()) != 0]
    if bad:
        raise SystemExit(f"device status {bad[0]} after the end-to-end steps")
    return {"value": res["M_all"] / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": n_e2e,
            "pipelined": "two input sets: step j+1's uploads overlap step j"}


def run_gpu(args):
    import gc

    import torch

    from pruned_expert_backward_lrmoe_b200 import inputs

    rank, world, local, dist = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks, peak_src = load_peaks()
    layer = inputs.make_layer(layer_spec(args), seed=args.seed)
    s = layer.spec
    res = measure_layer(layer, dev, args.steps, args.warmup, dist, peaks, peak_src)
    extras = run_extras(layer, res, dev, args, dist, peaks) if not args.no_extras and world == 1 else {}
    e2e = run_e2e(layer, res, dev, args, dist) if not args.no_extras else None

    # ---------------- CPU baseline (rank 0 at N = 1) ----------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        secs, m_cpu, experts = oracle_bounded_sample(layer, budget_s=args.cpu_budget)
        cpu = {"value": m_cpu / secs, "unit": UNIT, "cores": host_cores(), "kind": "oracle",
               "sample": f"{len(experts)} of the {s.E} experts of the {s.name} layer "
                         f"(experts {experts[0]}..{experts[-1]}, {m_cpu} retained pairs), each "
                         f"run as a standalone k=1 layer: score, selection, compaction, fp64 "
                         f"backward, unpack; {secs:.1f} s", **host_cpu()}

    # ---------------- the other configurations, after the headline ----------------
    others = {}
    if not args.no_extras and world == 1 and args.config == DEFAULT_CONFIG and not args.override:
        del res["runner"]
        gc.collect()
        torch.cuda.empty_cache()
        for name in OTHER_CONFIGS:
            lay = inputs.make_layer(inputs.spec(name), seed=args.seed)
            r = measure_layer(lay, dev, max(3, min(args.steps, 50)), max(3, args.warmup), dist,
                              peaks, peak_src)
            others[name] = {
                "workload": config_block(lay.spec, world)["workload"],
                "value": r["value"], "unit": UNIT, "ms_per_step": r["ms_per_step"],
                "retained_pairs": r["M"], "routed_pairs": lay.spec.P,
                "expert_bwd_tflops": r["expert_bwd_tflops"], "gemm_ms": r["gemm_ms"],
                "roofline": r["roofline"],
                "breakdown": {k_: {kk: v[kk] for kk in ("ms", "bound", "frac") if kk in v}
                              for k_, v in r["breakdown"].items()},
                "clocks": r["clocks"], "empty_experts": int((r["counts"] == 0).sum()),
            }
            del r, lay
            gc.collect()
            torch.cuda.empty_cache()

    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": s.dtype,
        "data": "synthetic", "config": config_block(s, world),
        "retained_pairs": res["M"], "routed_pairs": s.P,
        "expert_bwd_tflops": res["expert_bwd_tflops"], "gemm_ms": res["gemm_ms"],
        "roofline": res["roofline"], "breakdown": res["breakdown"],
        "breakdown_steps": res["breakdown_steps"], "breakdown_step_ms": res["breakdown_step_ms"],
        "cpu_baseline": cpu,
        "e2e": e2e if e2e is not None else {"value": None, "unit": UNIT, "h2d_bytes_per_step": 0,
                                            "d2h_bytes_per_step": 0},
        "gpu_launches": args.steps * sum(KERNEL_LAUNCHES.values()),
        "clocks": res["clocks"], "empty_experts": int((res["counts"] == 0).sum()),
        "peaks": {k_: peaks.get(k_) for k_ in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")},
        "peaks_source": peak_src,
        **extras,
        "other_configs": others,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_sweep(args):
    """Quota sweep on one GLM-shaped layer (T=16384): keep 4/4, 3/4, 2/4, 1/4 of every
    expert's pairs.  One JSON line per keep ratio (step time, grouped-GEMM TFLOP/s and
    their fraction of the bf16 peak), then a least-squares fit of step time against the
    retained pairs M (time should follow M, not the routed pairs P)."""
    import torch

    from pruned_expert_backward_lrmoe_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    base = inputs.spec(args.config if args.config.startswith("sweep") else "sweep100")
    layer = inputs.make_layer(base, seed=args.seed)
    s = layer.spec
    host, inp, out, stream, flush_l2, step = make_runner(layer, dev)
    peaks, peak_src = load_peaks()
    tf_peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    points = []
    for n in (4, 3, 2, 1):
        q = inputs.quota_from_counts(layer.counts, inputs.spec("sweep100", quota=f"keep:{n}/4"))
        inp["quota"].copy_(torch.from_numpy(q))
        out["status"].zero_()
        for _ in range(max(1, args.warmup)):
            step()
        torch.cuda.synchronize(dev)
        if int(out["status"].item()) != 0:
            raise SystemExit(f"device status {int(out['status'].item())} at keep {n}/4")
        M = int(out["offsets"][-1].item())
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(KERNELS) + 1)]
               for _ in range(args.steps)]
        with ClockSampler(0) as clk:
            for i in range(args.steps):
                flush_l2()
                step(evs[i])
            torch.cuda.synchronize(dev)
        kern = {kn: statistics.fmean(ev[j].elapsed_time(ev[j + 1]) for ev in evs)
                for j, kn in enumerate(KERNELS)}
        step_ms = statistics.fmean(ev[0].elapsed_time(ev[-1]) for ev in evs)
        by, fl = algorithmic(s.T, s.k, s.E, s.H, s.I, M, 2)
        gemm_ms = sum(kern[kn] for kn in step_gemms(fl))
        gemm_fl = sum(fl[kn] for kn in step_gemms(fl))
        tf = gemm_fl / (gemm_ms * 1e-3) / 1e12
        gemm_bytes = sum(by[kn] for kn in step_gemms(fl))
        points.append((M, step_ms))
        print(json.dumps({
            "sweep_keep": f"{n}/4", "retained_pairs": M, "routed_pairs": s.P,
            "ms_per_step": step_ms, "value": M / (step_ms * 1e-3), "unit": UNIT,
            "gemm_ms": gemm_ms, "gemm_tflops": tf, "gemm_tensor_frac": tf / tf_peak,
            "gemm_hbm_frac": gemm_bytes / (gemm_ms * 1e-3) / 1e9 / hbm_peak,
            "gemm_flop_per_byte": gemm_fl / gemm_bytes,
            "peaks": f"{peak_src}: bf16 {tf_peak} TFLOP/s sustained, HBM {hbm_peak} GB/s",
            "kernels_ms": kern, "clocks": clk.summary(), "steps": args.steps,
            "config": config_block(inputs.spec(f"sweep{25 * n}"), 1)}), flush=True)
    xs = np.array([p[0] for p in points], np.float64)
    ys = np.array([p[1] for p in points], np.float64)
    slope, intercept = np.polyfit(xs, ys, 1)
    resid = ys - (slope * xs + intercept)
    print(json.dumps({"sweep_fit": "ms_per_step = slope * M + intercept",
                      "slope_us_per_1k_pairs": slope * 1e6, "intercept_ms": intercept,
                      "max_abs_residual_ms": float(np.abs(resid).max()),
                      "routed_pairs": s.P}), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
