"""The C ABI library builds, loads without a GPU, exports every declared symbol,
and rejects host-detectable bad arguments before launching anything."""
import ctypes
import os
import re

import pytest

from pruned_expert_backward_lrmoe_b200 import build as B
from pruned_expert_backward_lrmoe_b200 import lrmoe as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "lrmoe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lrmoe_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(L.EXPORTS)


def test_checked_build_exports_the_same_symbols():
    """The checked-index debug library (-DLRMOE_CHECKED) builds and exports the
    same ABI; the binding selects it with LRMOE_CHECKED=1."""
    path = B.build(checked=True)
    assert path.endswith("liblrmoe_checked.so") and os.path.exists(path)
    chk = ctypes.CDLL(path)
    for n in declared_functions():
        assert hasattr(chk, n), n
    assert chk.lrmoe_version() == L.load().lrmoe_version()


def test_version_and_strings(lib):
    assert lib.lrmoe_version() >> 16 == 1
    assert lib.lrmoe_status_string(0) == b"ok"
    assert lib.lrmoe_status_string(4) == b"workspace too small"


def test_workspace_size_grows_with_pairs(lib):
    a = L.lrmoe_select_workspace_bytes(256, 2, 8)
    b = L.lrmoe_select_workspace_bytes(8192, 8, 128)
    assert 0 < a < b
    assert b >= 2 * 8192 * 8 * 4
    assert L.lrmoe_select_workspace_bytes(0, 8, 128) == 0


NULL = ctypes.c_void_p(0)
FAKE = ctypes.c_void_p(0x10000)  # aligned non-null; never dereferenced by the host checks


def test_score_rejects_bad_arguments(lib):
    f = lib.lrmoe_score
    # null pointer
    assert f(NULL, FAKE, 4, 2, 3, FAKE, 8, FAKE, 8, 1, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    assert b"topk_idx" in lib.lrmoe_last_error()
    # H not a multiple of 8 for bf16
    assert f(FAKE, FAKE, 4, 2, 3, FAKE, 12, FAKE, 8, 1, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    # misaligned pointer
    bad = ctypes.c_void_p(0x10004)
    assert f(FAKE, FAKE, 4, 2, 3, bad, 8, FAKE, 8, 1, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    # non-positive sizes, unknown dtype, k > 32
    assert f(FAKE, FAKE, 0, 2, 3, FAKE, 8, FAKE, 8, 1, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    assert f(FAKE, FAKE, 4, 2, 3, FAKE, 8, FAKE, 8, 7, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    assert f(FAKE, FAKE, 4, 33, 40, FAKE, 8, FAKE, 8, 1, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG


def test_row_norm_and_score_from_norms_reject_bad_arguments(lib):
    f = lib.lrmoe_row_sqnorm
    assert f(NULL, 4, 8, 1, FAKE, NULL) == L.LRMOE_ERR_INVALID_ARG
    assert b"rows" in lib.lrmoe_last_error()
    assert f(FAKE, 0, 8, 1, FAKE, NULL) == L.LRMOE_ERR_INVALID_ARG
    assert f(FAKE, 4, 12, 1, FAKE, NULL) == L.LRMOE_ERR_INVALID_ARG   # D % 8 for bf16
    assert f(FAKE, 4, 8, 5, FAKE, NULL) == L.LRMOE_ERR_INVALID_ARG    # dtype
    assert f(FAKE, 4, 8, 1, ctypes.c_void_p(0x10004), NULL) == L.LRMOE_ERR_INVALID_ARG
    g = lib.lrmoe_score_from_norms
    assert g(FAKE, FAKE, 4, 2, 3, FAKE, 8, NULL, 1, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    assert b"a_sqnorm" in lib.lrmoe_last_error()
    assert g(FAKE, FAKE, 4, 2, 3, FAKE, 6, FAKE, 0, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    assert g(FAKE, FAKE, 4, 33, 40, FAKE, 8, FAKE, 1, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    assert g(FAKE, FAKE, 4, 2, 0, FAKE, 8, FAKE, 1, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG


def test_router_grad_rejects_bad_arguments(lib):
    f = lib.lrmoe_router_grad
    assert f(FAKE, 4, 2, 3, FAKE, 8, NULL, 1, NULL, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    assert b"y_saved" in lib.lrmoe_last_error()
    assert f(FAKE, 4, 2, 3, FAKE, 8, FAKE, 1, ctypes.c_void_p(0x10004), FAKE, NULL, NULL) \
        == L.LRMOE_ERR_INVALID_ARG
    assert f(FAKE, 4, 2, 3, FAKE, 10, FAKE, 1, NULL, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    assert f(FAKE, 4, 0, 3, FAKE, 8, FAKE, 1, NULL, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG


def test_split_by_destination_rejects_bad_arguments(lib):
    f = lib.lrmoe_split_by_destination
    args = [FAKE, FAKE, FAKE, NULL, 4, 2, 100, FAKE, FAKE, FAKE, NULL, NULL, NULL]
    bad = list(args); bad[2] = NULL                       # plan
    assert f(*bad) == L.LRMOE_ERR_INVALID_ARG and b"plan" in lib.lrmoe_last_error()
    bad = list(args); bad[4] = 0                          # E
    assert f(*bad) == L.LRMOE_ERR_INVALID_ARG
    bad = list(args); bad[5] = 100000                     # G too large for shared memory
    assert f(*bad) == L.LRMOE_ERR_INVALID_ARG
    bad = list(args); bad[3] = ctypes.c_void_p(0x10004)   # misaligned global_start
    assert f(*bad) == L.LRMOE_ERR_INVALID_ARG


    bad = list(args); bad[10] = ctypes.c_void_p(0x10004)  # misaligned row_dest
    assert f(*bad) == L.LRMOE_ERR_INVALID_ARG and b"row_dest" in lib.lrmoe_last_error()


def test_group_received_rejects_bad_arguments(lib):
    f = lib.lrmoe_group_received
    args = [FAKE, 2, 4, 100, FAKE, FAKE, FAKE, NULL, NULL]
    bad = list(args); bad[0] = NULL
    assert f(*bad) == L.LRMOE_ERR_INVALID_ARG and b"src_expert_offsets" in lib.lrmoe_last_error()
    bad = list(args); bad[2] = 0                          # E
    assert f(*bad) == L.LRMOE_ERR_INVALID_ARG
    bad = list(args); bad[1] = 100000                     # G too large for shared memory
    assert f(*bad) == L.LRMOE_ERR_INVALID_ARG
    bad = list(args); bad[3] = 0                          # rows_cap
    assert f(*bad) == L.LRMOE_ERR_INVALID_ARG
    bad = list(args); bad[5] = NULL                       # inv
    assert f(*bad) == L.LRMOE_ERR_INVALID_ARG and b"inv" in lib.lrmoe_last_error()


def test_exchange_rows_reject_bad_arguments(lib):
    p = lib.lrmoe_pack_wide
    args = [FAKE, FAKE, FAKE, 4, 2, 3, FAKE, FAKE, 16, FAKE, FAKE, FAKE, 8, 1, FAKE, 8, NULL, NULL]
    bad = list(args); bad[10] = NULL                      # g
    assert p(*bad) == L.LRMOE_ERR_INVALID_ARG and b"g" in lib.lrmoe_last_error()
    bad = list(args); bad[12] = 12                        # I not a multiple of 8 (bf16)
    assert p(*bad) == L.LRMOE_ERR_INVALID_ARG
    bad = list(args); bad[15] = 0                         # rows_cap
    assert p(*bad) == L.LRMOE_ERR_INVALID_ARG
    s = lib.lrmoe_split_wide
    args = [FAKE, 10, FAKE, 4, 16, 8, 1, FAKE, FAKE, FAKE, FAKE, FAKE, NULL, NULL]
    bad = list(args); bad[11] = NULL                      # Up
    assert s(*bad) == L.LRMOE_ERR_INVALID_ARG and b"Up" in lib.lrmoe_last_error()
    bad = list(args); bad[1] = 0                          # n_src
    assert s(*bad) == L.LRMOE_ERR_INVALID_ARG
    bad = list(args); bad[3] = 0                          # nothing to do
    assert s(*bad) == L.LRMOE_OK


def test_fused_gemm_rejects_bad_arguments(lib):
    f = lib.lrmoe_grouped_dgrad_wgrad
    args = [FAKE, 64, FAKE, FAKE, 4, 64, 64, 1, 0, NULL, NULL, FAKE, FAKE, 64, FAKE, 0, NULL, NULL]
    bad = list(args); bad[7] = 0                          # fp32: the fused launch is bf16 only
    assert f(*bad) == L.LRMOE_ERR_UNSUPPORTED
    bad = list(args); bad[14] = NULL                      # dW
    assert f(*bad) == L.LRMOE_ERR_INVALID_ARG and b"dW" in lib.lrmoe_last_error()
    bad = list(args); bad[8] = 1                          # SwiGLU epilogue without g, u
    assert f(*bad) == L.LRMOE_ERR_INVALID_ARG
    bad = list(args); bad[13] = 12                        # N2 not a multiple of 8
    assert f(*bad) == L.LRMOE_ERR_INVALID_ARG
    bad = list(args); bad[4] = 5000                       # E above the grouped-GEMM limit
    assert f(*bad) == L.LRMOE_ERR_UNSUPPORTED


def test_gather_rows_rejects_bad_arguments(lib):
    f = lib.lrmoe_gather_rows
    assert f(FAKE, 10, 24, FAKE, 4, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG  # 24 % 16
    assert f(NULL, 10, 32, FAKE, 4, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    assert f(FAKE, 0, 32, FAKE, 4, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    assert f(FAKE, 10, 32, FAKE, 0, FAKE, NULL, NULL) == L.LRMOE_OK              # nothing to do


def test_select_rejects_small_workspace(lib):
    f = lib.lrmoe_select_quota
    need = L.lrmoe_select_workspace_bytes(64, 2, 4)
    ws = ctypes.c_void_p(0x100000)
    r = f(FAKE, FAKE, 64, 2, 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws, need - 1, NULL, NULL)
    assert r == L.LRMOE_ERR_WORKSPACE
    r = f(FAKE, FAKE, 64, 2, 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_void_p(0x100010),
          need, NULL, NULL)
    assert r == L.LRMOE_ERR_WORKSPACE       # not 256-byte aligned
    r = f(FAKE, FAKE, 64, 2, 5000, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws, 1 << 30, NULL, NULL)
    assert r == L.LRMOE_ERR_UNSUPPORTED     # E > 4096


def test_gemm_rejects_bad_arguments(lib):
    d = lib.lrmoe_grouped_dgrad
    # unknown epilogue
    assert d(FAKE, 16, FAKE, FAKE, 2, 64, 64, 1, 9, NULL, NULL, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    # SwiGLU epilogue needs g and u
    assert d(FAKE, 16, FAKE, FAKE, 2, 64, 64, 1, 1, NULL, NULL, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    # too many experts for the tile table
    assert d(FAKE, 16, FAKE, FAKE, 2000, 64, 64, 1, 0, NULL, NULL, FAKE, NULL, NULL) == L.LRMOE_ERR_UNSUPPORTED
    w = lib.lrmoe_grouped_wgrad
    assert w(FAKE, FAKE, 16, FAKE, 2, 60, 64, 1, FAKE, 0, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    assert w(FAKE, FAKE, 16, NULL, 2, 64, 64, 1, FAKE, 0, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG


def test_pack_unpack_reject_bad_arguments(lib):
    p = lib.lrmoe_pack
    assert p(FAKE, FAKE, FAKE, 4, 2, 3, FAKE, FAKE, 8, FAKE, FAKE, FAKE, 8, 1, FAKE, FAKE, FAKE,
             FAKE, NULL, 8, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    assert p(FAKE, FAKE, FAKE, 4, 2, 3, FAKE, FAKE, 8, FAKE, FAKE, FAKE, 8, 1, FAKE, FAKE, FAKE,
             FAKE, FAKE, 0, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    u = lib.lrmoe_unpack
    assert u(FAKE, 8, FAKE, 4, 2, 6, 0, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG  # H % 4
    assert u(FAKE, 8, NULL, 4, 2, 8, 0, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG


def test_pruned_backward_rejects_null_struct(lib):
    assert lib.lrmoe_pruned_backward(None, 4, 2, 3, 8, 8, 8, 1, NULL) == L.LRMOE_ERR_INVALID_ARG


def test_selftest_rejects_bad_arguments(lib):
    f = lib.lrmoe_selftest_bounded_wait
    assert f(0, FAKE, NULL) == L.LRMOE_ERR_INVALID_ARG
    assert f(2_000_000, FAKE, NULL) == L.LRMOE_ERR_INVALID_ARG
    assert f(100, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG


def test_quota_controller_rejects_bad_arguments(lib):
    f = lib.lrmoe_quota_controller
    assert f(NULL, 4, 2, 3, 0, -1, FAKE, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG
    assert f(FAKE, 4, 2, 5000, 0, -1, FAKE, FAKE, NULL, NULL) == L.LRMOE_ERR_UNSUPPORTED
    assert f(FAKE, 0, 2, 3, 0, -1, FAKE, FAKE, NULL, NULL) == L.LRMOE_ERR_INVALID_ARG


def test_binding_selects_the_checked_library_by_environment():
    """LRMOE_CHECKED=1 makes the binding load liblrmoe_checked.so (read once, at import)."""
    import subprocess
    import sys
    code = ("from pruned_expert_backward_lrmoe_b200 import lrmoe as L; "
            "print(L.LIB_PATH.rsplit('/', 1)[-1])")
    for env_val, want in (("1", "liblrmoe_checked.so"), (None, "liblrmoe.so")):
        env = dict(os.environ)
        env.pop("LRMOE_CHECKED", None)
        if env_val is not None:
            env["LRMOE_CHECKED"] = env_val
        r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True,
                           text=True, timeout=300)
        assert r.returncode == 0, r.stderr[-2000:]
        assert r.stdout.strip() == want
