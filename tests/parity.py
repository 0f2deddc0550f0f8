"""Shared helpers of the GPU parity tests: device copies of a generated layer,
the CUDA path through the C ABI, and element-by-element comparison with the
CPU oracle.

Tolerances (relative Frobenius error of each gradient tensor against the
fp64 oracle, worst expert reported): 1e-5 for fp32 storage, 2e-2 for bf16
storage with fp32 accumulation.  Selection, packing and scores: bit-exact.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import lrmoe_oracle as O
from pruned_expert_backward_lrmoe_b200 import lrmoe as L

TOL = {"f32": 1e-5, "bf16": 2e-2}


def storage_tensor(arr: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).to(device)


def to_numpy_storage(t: torch.Tensor, dtype: str) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if dtype == "bf16":
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def device_inputs(layer, device="cuda"):
    dt = layer.dtype
    return {
        "topk_idx": torch.from_numpy(layer.topk_idx).to(device),
        "topk_w": torch.from_numpy(layer.topk_w).to(device),
        "quota": torch.from_numpy(layer.quota).to(device),
        "x": storage_tensor(layer.x, dt, device),
        "dY": storage_tensor(layer.dY, dt, device),
        "g": storage_tensor(layer.g, dt, device),
        "u": storage_tensor(layer.u, dt, device),
        "a": storage_tensor(layer.a, dt, device),
        "W_gu": storage_tensor(layer.W_gu, dt, device),
        "W_down": storage_tensor(layer.W_down, dt, device),
    }


def run_steps(layer, inp=None, poison=True, out=None):
    """Run a1..a5 one entry point at a time; returns the device buffers (`out`:
    buffers laid out like alloc_buffers' to use instead of fresh ones)."""
    s = layer.spec
    tdt = torch.bfloat16 if s.dtype == "bf16" else torch.float32
    inp = inp or device_inputs(layer)
    if out is None:
        out = L.alloc_buffers(s.T, s.k, s.E, s.H, s.I, tdt)
    if poison:  # unwritten memory must not leak into results
        for k_, v in out.items():
            if k_ in ("status",):
                continue
            if v.dtype in (torch.float32, torch.bfloat16):
                v.fill_(float("nan"))
            elif v.dtype == torch.int32:
                v.fill_(-7)
            else:
                v.fill_(0xAB)
    out["status"].zero_()
    st = out["status"]
    L.lrmoe_score(inp["topk_idx"], inp["topk_w"], inp["dY"], inp["a"], s.E, out["score"], st)
    L.lrmoe_select_quota(inp["topk_idx"], out["score"], inp["quota"], out["counts"], out["kept"],
                         out["offsets"], out["perm"], out["pos"], out["workspace"], st)
    L.lrmoe_pack(out["perm"], out["offsets"], inp["topk_w"], inp["x"], inp["dY"], inp["a"],
                 inp["g"], inp["u"], out["Xp"], out["DYp"], out["Ap"], out["Gp"], out["Up"], st)
    L.lrmoe_grouped_dgrad(out["DYp"], inp["W_down"], out["offsets"], L.LRMOE_EPI_SWIGLU_BWD,
                          out["dGUp"], Gp=out["Gp"], Up=out["Up"], status=st)
    L.lrmoe_grouped_wgrad(out["DYp"], out["Ap"], out["offsets"], out["dW_down"], status=st)
    L.lrmoe_grouped_wgrad(out["dGUp"], out["Xp"], out["offsets"], out["dW_gu"], status=st)
    L.lrmoe_grouped_dgrad(out["dGUp"], inp["W_gu"], out["offsets"], L.LRMOE_EPI_STORE, out["dXp"],
                          status=st)
    L.lrmoe_unpack(out["dXp"], out["pos"], s.T, s.k, out["dX"], st)
    torch.cuda.synchronize()
    return out


def run_chain(layer, inp=None, out=None):
    s = layer.spec
    tdt = torch.bfloat16 if s.dtype == "bf16" else torch.float32
    inp = inp or device_inputs(layer)
    if out is None:
        out = L.alloc_buffers(s.T, s.k, s.E, s.H, s.I, tdt)
    out["status"].zero_()
    L.lrmoe_pruned_backward(inp, out)
    torch.cuda.synchronize()
    return out


def rel_fro(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    d = np.linalg.norm(b)
    if d == 0:
        return 0.0 if np.linalg.norm(a) == 0 else np.inf
    return float(np.linalg.norm(a - b) / d)


def check_selection(layer, out, ref):
    """score, counts, kept, offsets, perm, pos: bit-exact."""
    np.testing.assert_array_equal(out["score"].cpu().numpy().view(np.uint32),
                                  ref["score"].view(np.uint32))
    for name in ("counts", "kept", "offsets", "pos"):
        np.testing.assert_array_equal(out[name].cpu().numpy(), ref[name], err_msg=name)
    M = int(ref["offsets"][-1])
    np.testing.assert_array_equal(out["perm"].cpu().numpy()[:M], ref["perm"], err_msg="perm")
    return M


def chain_packed(layer):
    """Packed buffers the chain entry point writes: for bf16 the SwiGLU epilogue reads
    g, u in place (at row perm[r]), so G_p and U_p are not packed."""
    return ("Xp", "DYp", "Ap") if layer.dtype == "bf16" else ("Xp", "DYp", "Ap", "Gp", "Up")


def check_pack(layer, out, ref, M, names=("Xp", "DYp", "Ap", "Gp", "Up")):
    dt = layer.dtype
    for name in names:
        got = to_numpy_storage(out[name][:M], dt)
        np.testing.assert_array_equal(got, np.asarray(ref[name]), err_msg=name)


def check_gradients(layer, out, ref, experts=None):
    """dW_down, dW_gu per expert and dX within tolerance; m_e = 0 experts exactly zero."""
    dt = layer.dtype
    tol = TOL[dt]
    E = layer.spec.E
    kept = ref["kept"]
    sel = range(E) if experts is None else experts
    dWd = out["dW_down"].cpu().numpy()
    dWgu = out["dW_gu"].cpu().numpy()
    worst = {"dW_down": 0.0, "dW_gu": 0.0}
    for e in sel:
        for name, got in (("dW_down", dWd[e]), ("dW_gu", dWgu[e])):
            want = ref[name][e]
            if kept[e] == 0:
                assert not got.any(), f"{name}[{e}] must be exactly zero"
                continue
            err = rel_fro(got, want)
            worst[name] = max(worst[name], err)
            assert err <= tol, f"{name}[{e}] rel err {err:.3e} > {tol}"
    if experts is None:
        assert rel_fro(dWd, ref["dW_down"]) <= tol
        assert rel_fro(dWgu, ref["dW_gu"]) <= tol
    dX = out["dX"].float().cpu().numpy()
    err = rel_fro(dX, ref["dX"])
    assert err <= tol, f"dX rel err {err:.3e} > {tol}"
    none = (ref["pos"].reshape(layer.spec.T, layer.spec.k) < 0).all(axis=1)
    assert not dX[none].any(), "tokens with no retained pair must get dX = 0"
    worst["dX"] = err
    return worst
