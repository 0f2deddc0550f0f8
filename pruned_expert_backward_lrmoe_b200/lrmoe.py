"""ctypes binding of liblrmoe.so (the C ABI in include/lrmoe.h).

Functions carry the C names and only marshal arguments: torch tensors become
device pointers, the current torch stream becomes the cudaStream_t.  Every
step of the path runs in the library's CUDA kernels; there is no fallback.
If the library is missing, the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# LRMOE_CHECKED=1 selects the checked-index debug build (see build.py --checked)
LIB_PATH = os.path.join(_HERE, "liblrmoe_checked.so" if os.environ.get("LRMOE_CHECKED") == "1"
                        else "liblrmoe.so")

LRMOE_OK, LRMOE_ERR_INVALID_ARG, LRMOE_ERR_UNSUPPORTED, LRMOE_ERR_CUDA, LRMOE_ERR_WORKSPACE = range(5)
LRMOE_F32, LRMOE_BF16 = 0, 1
LRMOE_EPI_STORE, LRMOE_EPI_SWIGLU_BWD = 0, 1
ST_BAD_EXPERT, ST_BAD_QUOTA, ST_NONFINITE, ST_TIMEOUT, ST_BAD_INDEX = 1, 2, 4, 8, 16

# every symbol the header declares
EXPORTS = ("lrmoe_version", "lrmoe_status_string", "lrmoe_last_error", "lrmoe_score",
           "lrmoe_select_workspace_bytes", "lrmoe_select_quota", "lrmoe_pack",
           "lrmoe_grouped_dgrad", "lrmoe_grouped_wgrad", "lrmoe_unpack", "lrmoe_pruned_backward",
           "lrmoe_select_quota_noalloc", "lrmoe_selftest_bounded_wait", "lrmoe_quota_controller",
           "lrmoe_row_sqnorm", "lrmoe_score_from_norms", "lrmoe_router_grad",
           "lrmoe_redistribute", "lrmoe_split_by_destination", "lrmoe_grouped_dgrad_wgrad",
           "lrmoe_grouped_dgrad_swiglu_gather", "lrmoe_grouped_wgrad_gather", "lrmoe_gather_rows",
           "lrmoe_group_received", "lrmoe_pack_wide", "lrmoe_split_wide",
           "lrmoe_selftest_gemm_stall")
NOALLOC_SCRATCH_BYTES = 4 << 20


class LrmoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"lrmoe error {code}: {msg}")
        self.code = code


class lrmoe_buffers(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "topk_idx", "topk_w", "quota", "x", "dY", "g", "u", "a", "W_gu", "W_down",
        "score", "counts", "kept", "offsets", "perm", "pos",
        "Xp", "DYp", "Ap", "Gp", "Up", "dGUp", "dXp", "dW_gu", "dW_down", "dX",
        "workspace")] + [("workspace_bytes", ctypes.c_size_t), ("status", ctypes.c_void_p)]


_lib: Optional[ctypes.CDLL] = None


def load() -> ctypes.CDLL:
    """Load liblrmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m pruned_expert_backward_lrmoe_b200.build`"
                           + (" --checked" if LIB_PATH.endswith("_checked.so") else ""))
    lib = ctypes.CDLL(LIB_PATH)
    P, I, Z, U32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint32
    lib.lrmoe_version.restype = I
    lib.lrmoe_status_string.restype = ctypes.c_char_p
    lib.lrmoe_status_string.argtypes = [I]
    lib.lrmoe_last_error.restype = ctypes.c_char_p
    lib.lrmoe_score.argtypes = [P, P, I, I, I, P, I, P, I, I, P, P, P]
    lib.lrmoe_row_sqnorm.argtypes = [P, I, I, I, P, P]
    lib.lrmoe_router_grad.argtypes = [P, I, I, I, P, I, P, I, P, P, P, P]
    lib.lrmoe_redistribute.argtypes = [P, P, I, I, P, P]
    lib.lrmoe_split_by_destination.argtypes = [P, P, P, P, I, I, I, P, P, P, P, P, P]
    lib.lrmoe_group_received.argtypes = [P, I, I, I, P, P, P, P, P]
    lib.lrmoe_pack_wide.argtypes = [P, P, P, I, I, I, P, P, I, P, P, P, I, I, P, I, P, P]
    lib.lrmoe_split_wide.argtypes = [P, I, P, I, I, I, I, P, P, P, P, P, P, P]
    lib.lrmoe_score_from_norms.argtypes = [P, P, I, I, I, P, I, P, I, P, P, P]
    lib.lrmoe_select_workspace_bytes.argtypes = [I, I, I]
    lib.lrmoe_select_workspace_bytes.restype = Z
    lib.lrmoe_select_quota.argtypes = [P, P, I, I, I, P, P, P, P, P, P, P, Z, P, P]
    lib.lrmoe_select_quota_noalloc.argtypes = [P, P, I, I, I, P, P, P, P, P, P, P, P]
    lib.lrmoe_selftest_bounded_wait.argtypes = [U32, P, P]
    lib.lrmoe_selftest_gemm_stall.argtypes = [P, I, P, P, I, I, I, P, I, U32, P, P]
    lib.lrmoe_quota_controller.argtypes = [P, I, I, I, ctypes.c_int32, ctypes.c_int64, P, P, P, P]
    lib.lrmoe_pack.argtypes = [P, P, P, I, I, I, P, P, I, P, P, P, I, I, P, P, P, P, P, I, P, P]
    lib.lrmoe_grouped_dgrad.argtypes = [P, I, P, P, I, I, I, I, I, P, P, P, P, P]
    lib.lrmoe_grouped_wgrad.argtypes = [P, P, I, P, I, I, I, I, P, I, P, P]
    lib.lrmoe_grouped_dgrad_swiglu_gather.argtypes = [P, I, P, P, I, I, I, I, P, P, P, I, P, P, P]
    lib.lrmoe_grouped_wgrad_gather.argtypes = [P, I, P, P, I, I, P, I, I, I, I, P, I, P, P]
    lib.lrmoe_gather_rows.argtypes = [P, I, I, P, I, P, P, P]
    lib.lrmoe_grouped_dgrad_wgrad.argtypes = [P, I, P, P, I, I, I, I, I, P, P, P, P, I, P, I, P, P]
    lib.lrmoe_unpack.argtypes = [P, I, P, I, I, I, I, P, P, P]
    lib.lrmoe_pruned_backward.argtypes = [ctypes.POINTER(lrmoe_buffers), I, I, I, I, I, I, I, P]
    _lib = lib
    return lib


def _check(code: int) -> None:
    if code != LRMOE_OK:
        msg = load().lrmoe_last_error().decode()
        raise LrmoeError(code, msg or load().lrmoe_status_string(code).decode())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return LRMOE_BF16
    if t.dtype == torch.float32:
        return LRMOE_F32
    raise ValueError(f"unsupported storage dtype {t.dtype}")


# ---------------------------------------------------------------------------
# one function per C entry point
# ---------------------------------------------------------------------------
def lrmoe_version() -> int:
    return load().lrmoe_version()


def lrmoe_select_workspace_bytes(T: int, k: int, E: int) -> int:
    return int(load().lrmoe_select_workspace_bytes(T, k, E))


def lrmoe_score(topk_idx, topk_w, dY, a_saved, E: int, score, status=None, stream=None) -> None:
    T, k = topk_idx.shape
    _check(load().lrmoe_score(_ptr(topk_idx), _ptr(topk_w), T, k, E, _ptr(dY), dY.shape[-1],
                              _ptr(a_saved), a_saved.shape[-1], _dt(dY), _ptr(score), _ptr(status),
                              _stream(stream)))


def lrmoe_row_sqnorm(rows, out, stream=None) -> None:
    """out[r] = ||rows[r]||^2 (canonical order) for every row of a 2-D tensor."""
    _check(load().lrmoe_row_sqnorm(_ptr(rows), rows.shape[0], rows.shape[-1], _dt(rows), _ptr(out),
                                   _stream(stream)))


def lrmoe_score_from_norms(topk_idx, topk_w, dY, a_sqnorm, E: int, score, status=None,
                           stream=None) -> None:
    T, k = topk_idx.shape
    _check(load().lrmoe_score_from_norms(_ptr(topk_idx), _ptr(topk_w), T, k, E, _ptr(dY),
                                         dY.shape[-1], _ptr(a_sqnorm), _dt(dY), _ptr(score),
                                         _ptr(status), _stream(stream)))


def lrmoe_router_grad(topk_idx, dY, y_saved, E: int, dw, pos=None, status=None,
                      stream=None) -> None:
    """dw[p] = <dY_t, y_p> for routed pairs (retained pairs only when pos is given)."""
    T, k = topk_idx.shape
    _check(load().lrmoe_router_grad(_ptr(topk_idx), T, k, E, _ptr(dY), dY.shape[-1],
                                    _ptr(y_saved), _dt(dY), _ptr(pos), _ptr(dw), _ptr(status),
                                    _stream(stream)))


def lrmoe_redistribute(m, admissible):
    """Host planner: (plan [E][G] int64, peak) for retained counts m [E] and the
    copy map admissible [E][G] (numpy or CPU tensors)."""
    import numpy as np
    m = np.ascontiguousarray(np.asarray(m), dtype=np.int64)
    adm = np.ascontiguousarray(np.asarray(admissible) != 0, dtype=np.uint8)
    E, G = adm.shape
    plan = np.zeros((E, G), dtype=np.int64)
    peak = np.zeros(1, dtype=np.int64)
    _check(load().lrmoe_redistribute(m.ctypes.data, adm.ctypes.data, E, G, plan.ctypes.data,
                                     peak.ctypes.data))
    return plan, int(peak[0])


def lrmoe_split_by_destination(perm, offsets, plan, perm_dest, dest_offsets, dest_expert_offsets,
                               global_start=None, status=None, stream=None,
                               row_dest=None) -> None:
    E, G = plan.shape
    _check(load().lrmoe_split_by_destination(_ptr(perm), _ptr(offsets), _ptr(plan),
                                             _ptr(global_start), E, G, perm.shape[0],
                                             _ptr(perm_dest), _ptr(dest_offsets),
                                             _ptr(dest_expert_offsets), _ptr(row_dest),
                                             _ptr(status), _stream(stream)))


def lrmoe_group_received(src_expert_offsets, order, inv, offsets, status=None,
                         stream=None) -> None:
    """Received rows (source-major) regrouped expert-major: order, inv, offsets."""
    G, E1 = src_expert_offsets.shape
    _check(load().lrmoe_group_received(_ptr(src_expert_offsets), G, E1 - 1, order.numel(),
                                       _ptr(order), _ptr(inv), _ptr(offsets), _ptr(status),
                                       _stream(stream)))


def lrmoe_pack_wide(perm, offsets, topk_w, x, dY, a, g, u, rows, status=None, stream=None) -> None:
    """rows[r] = [x_t | RNE(w_p dY_t) | a_p | g_p | u_p] for packed rows r < offsets[-1]."""
    T, k = topk_w.shape
    E = offsets.numel() - 1
    _check(load().lrmoe_pack_wide(_ptr(perm), _ptr(offsets), _ptr(topk_w), T, k, E, _ptr(x),
                                  _ptr(dY), dY.shape[-1], _ptr(a), _ptr(g), _ptr(u), a.shape[-1],
                                  _dt(dY), _ptr(rows), rows.shape[0], _ptr(status),
                                  _stream(stream)))


def lrmoe_split_wide(rows, idx, Xp, DYp, Ap, Gp, Up, status=None, stream=None) -> None:
    """The five column blocks of rows[idx[i]] into X_p[i], DY_p[i], A_p[i], G_p[i], U_p[i]."""
    n = idx.numel()
    if n == 0:
        return
    _check(load().lrmoe_split_wide(_ptr(rows), rows.shape[0], _ptr(idx), n, Xp.shape[-1],
                                   Ap.shape[-1], _dt(Xp), _ptr(Xp), _ptr(DYp), _ptr(Ap), _ptr(Gp),
                                   _ptr(Up), _ptr(status), _stream(stream)))


def lrmoe_select_quota(topk_idx, score, quota, counts, kept, offsets, perm, pos, workspace,
                       status=None, stream=None) -> None:
    T, k = topk_idx.shape
    E = quota.numel()
    _check(load().lrmoe_select_quota(_ptr(topk_idx), _ptr(score), T, k, E, _ptr(quota),
                                     _ptr(counts), _ptr(kept), _ptr(offsets), _ptr(perm),
                                     _ptr(pos), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _ptr(status), _stream(stream)))


def lrmoe_quota_controller(topk_idx, E: int, cap: int, max_pairs: int, quota, counts, status=None,
                           stream=None) -> None:
    """Per-expert quotas on the device: min(count, cap, tau) with tau the largest level
    whose total fits max_pairs (cap <= 0 / max_pairs < 0 disable the limits)."""
    T, k = topk_idx.shape
    _check(load().lrmoe_quota_controller(_ptr(topk_idx), T, k, E, int(cap), int(max_pairs),
                                         _ptr(quota), _ptr(counts), _ptr(status), _stream(stream)))


def lrmoe_select_quota_noalloc(topk_idx, score, quota, counts, kept, offsets, perm, pos,
                               status=None, stream=None) -> None:
    """Selection without a workspace, for callers that cannot allocate device scratch.

    The library's own fixed scratch array (NOALLOC_SCRATCH_BYTES per GPU) is used
    instead; calls that overlap on the GPU race on it.
    """
    T, k = topk_idx.shape
    E = quota.numel()
    _check(load().lrmoe_select_quota_noalloc(_ptr(topk_idx), _ptr(score), T, k, E, _ptr(quota),
                                             _ptr(counts), _ptr(kept), _ptr(offsets), _ptr(perm),
                                             _ptr(pos), _ptr(status), _stream(stream)))


def lrmoe_pack(perm, offsets, topk_w, x, dY, a, g, u, Xp, DYp, Ap, Gp, Up, status=None,
               stream=None, I: Optional[int] = None) -> None:
    """Only dY/DYp are required; x/Xp, a/Ap and g, u/Gp, Up may be None (not packed)."""
    T, k = topk_w.shape
    E = offsets.numel() - 1
    if I is None:
        feat = next((t for t in (a, g, u, Ap, Gp, Up) if t is not None), None)
        I = feat.shape[-1] if feat is not None else 8
    _check(load().lrmoe_pack(_ptr(perm), _ptr(offsets), _ptr(topk_w), T, k, E, _ptr(x), _ptr(dY),
                             dY.shape[-1], _ptr(a), _ptr(g), _ptr(u), I, _dt(dY), _ptr(Xp),
                             _ptr(DYp), _ptr(Ap), _ptr(Gp), _ptr(Up), DYp.shape[0], _ptr(status),
                             _stream(stream)))


def lrmoe_grouped_dgrad(rows, W, offsets, epilogue: int, out, Gp=None, Up=None, status=None,
                        stream=None) -> None:
    E, K, N = W.shape
    _check(load().lrmoe_grouped_dgrad(_ptr(rows), rows.shape[0], _ptr(W), _ptr(offsets), E, K, N,
                                      _dt(rows), epilogue, _ptr(Gp), _ptr(Up), _ptr(out),
                                      _ptr(status), _stream(stream)))


def lrmoe_grouped_wgrad(grad_rows, in_rows, offsets, dW, accumulate: bool = False, status=None,
                        stream=None) -> None:
    E, N1, N2 = dW.shape
    _check(load().lrmoe_grouped_wgrad(_ptr(grad_rows), _ptr(in_rows), grad_rows.shape[0],
                                      _ptr(offsets), E, N1, N2, _dt(grad_rows), _ptr(dW),
                                      int(accumulate), _ptr(status), _stream(stream)))


def lrmoe_grouped_dgrad_swiglu_gather(rows, W, offsets, perm, g, u, out, status=None,
                                      stream=None) -> None:
    """dgrad with the SwiGLU-backward epilogue reading g, u [T*k][N] at row perm[r] (bf16)."""
    E, K, N = W.shape
    _check(load().lrmoe_grouped_dgrad_swiglu_gather(_ptr(rows), rows.shape[0], _ptr(W),
                                                    _ptr(offsets), E, K, N, _dt(rows), _ptr(perm),
                                                    _ptr(g), _ptr(u), g.shape[0], _ptr(out),
                                                    _ptr(status), _stream(stream)))


def lrmoe_grouped_wgrad_gather(grad_rows, perm, src, src_div: int, n_pairs: int, offsets, dW,
                               accumulate: bool = False, status=None, stream=None) -> None:
    """dW[e] = grad[R_e]^T . src[perm[r] / src_div] rows (bf16)."""
    E, N1, N2 = dW.shape
    _check(load().lrmoe_grouped_wgrad_gather(_ptr(grad_rows), grad_rows.shape[0], _ptr(perm),
                                             _ptr(src), int(src_div), int(n_pairs), _ptr(offsets),
                                             E, N1, N2, _dt(grad_rows), _ptr(dW), int(accumulate),
                                             _ptr(status), _stream(stream)))


def lrmoe_gather_rows(src, idx, dst, status=None, stream=None) -> None:
    """dst[i] = src[idx[i]] for the rows of 2-D tensors (row bytes a multiple of 16)."""
    n = idx.numel()
    if n == 0:
        return
    _check(load().lrmoe_gather_rows(_ptr(src), src.shape[0], src.shape[1] * src.element_size(),
                                    _ptr(idx), n, _ptr(dst), _ptr(status), _stream(stream)))


def lrmoe_grouped_dgrad_wgrad(grad_rows, W, offsets, epilogue: int, out, in_rows, dW, Gp=None,
                              Up=None, accumulate: bool = False, status=None,
                              stream=None) -> None:
    """lrmoe_grouped_dgrad(grad_rows, W, ...) and lrmoe_grouped_wgrad(grad_rows, in_rows, dW)
    in one launch (bf16)."""
    E, K, N = W.shape
    _check(load().lrmoe_grouped_dgrad_wgrad(_ptr(grad_rows), grad_rows.shape[0], _ptr(W),
                                            _ptr(offsets), E, K, N, _dt(grad_rows), epilogue,
                                            _ptr(Gp), _ptr(Up), _ptr(out), _ptr(in_rows),
                                            in_rows.shape[-1], _ptr(dW), int(accumulate),
                                            _ptr(status), _stream(stream)))


def lrmoe_unpack(dXp, pos, T: int, k: int, dX, status=None, stream=None) -> None:
    _check(load().lrmoe_unpack(_ptr(dXp), dXp.shape[0], _ptr(pos), T, k, dXp.shape[-1], _dt(dXp),
                               _ptr(dX), _ptr(status), _stream(stream)))


def lrmoe_selftest_gemm_stall(rows, W, offsets, out, two_sm: bool, limit_us: int, status,
                              stream=None) -> None:
    """The grouped dgrad with its first K block withheld; must set ST_TIMEOUT."""
    E, K, N = W.shape
    _check(load().lrmoe_selftest_gemm_stall(_ptr(rows), rows.shape[0], _ptr(W), _ptr(offsets), E,
                                            K, N, _ptr(out), int(bool(two_sm)), int(limit_us),
                                            _ptr(status), _stream(stream)))


def lrmoe_selftest_bounded_wait(limit_us: int, status, stream=None) -> None:
    """Run one device wait that must give up after `limit_us` and set ST_TIMEOUT."""
    _check(load().lrmoe_selftest_bounded_wait(int(limit_us), _ptr(status), _stream(stream)))


# ---------------------------------------------------------------------------
# whole path
# ---------------------------------------------------------------------------
def alloc_buffers(T: int, k: int, E: int, H: int, I: int, dtype: torch.dtype,
                  device="cuda", rows_cap: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Device buffers for every output and intermediate of lrmoe_pruned_backward."""
    P = T * k
    R = P if rows_cap is None else rows_cap
    i32 = dict(dtype=torch.int32, device=device)
    st = dict(dtype=dtype, device=device)
    ws_bytes = lrmoe_select_workspace_bytes(T, k, E)
    return {
        "score": torch.empty(P, dtype=torch.float32, device=device),
        "counts": torch.empty(E, **i32), "kept": torch.empty(E, **i32),
        "offsets": torch.empty(E + 1, **i32), "perm": torch.empty(P, **i32),
        "pos": torch.empty(P, **i32),
        "Xp": torch.empty(R, H, **st), "DYp": torch.empty(R, H, **st),
        "Ap": torch.empty(R, I, **st), "Gp": torch.empty(R, I, **st), "Up": torch.empty(R, I, **st),
        "dGUp": torch.empty(R, 2 * I, **st), "dXp": torch.empty(R, H, **st),
        "dW_gu": torch.empty(E, 2 * I, H, dtype=torch.float32, device=device),
        "dW_down": torch.empty(E, H, I, dtype=torch.float32, device=device),
        "dX": torch.empty(T, H, **st),
        "workspace": torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=device),
        "status": torch.zeros(1, dtype=torch.int32, device=device),
    }


def lrmoe_pruned_backward(inp: Dict[str, torch.Tensor], out: Dict[str, torch.Tensor],
                          stream=None) -> None:
    """Enqueue a1..a5 for one layer.  `inp`: topk_idx, topk_w, quota, x, dY, g, u, a, W_gu, W_down."""
    T, k = inp["topk_idx"].shape
    E, H, I = inp["W_down"].shape
    b = lrmoe_buffers()
    for name in ("topk_idx", "topk_w", "quota", "x", "dY", "g", "u", "a", "W_gu", "W_down"):
        setattr(b, name, _ptr(inp[name]))
    for name in ("score", "counts", "kept", "offsets", "perm", "pos", "Xp", "DYp", "Ap", "Gp",
                 "Up", "dGUp", "dXp", "dW_gu", "dW_down", "dX", "workspace", "status"):
        setattr(b, name, _ptr(out[name]))
    b.workspace_bytes = out["workspace"].numel()
    _check(load().lrmoe_pruned_backward(ctypes.byref(b), T, k, E, H, I, out["Xp"].shape[0],
                                        _dt(inp["x"]), _stream(stream)))
