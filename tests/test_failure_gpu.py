"""Failure detection on the GPU without a fault: a bounded device wait on a
barrier that nothing completes must give up, report LRMOE_ST_TIMEOUT in the
status word and leave the context usable for the next call."""
import time

import pytest
import torch

from pruned_expert_backward_lrmoe_b200 import inputs
from pruned_expert_backward_lrmoe_b200 import lrmoe as L

from tests import parity as PT

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    L.lrmoe_selftest_bounded_wait(2000, status)     # 2 ms limit
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    st = int(status.item())
    assert st & L.ST_TIMEOUT
    assert not st & L.ST_BAD_INDEX                   # the wait never "succeeded"
    assert elapsed < 1.0
    # the context still runs the real path correctly afterwards
    layer = inputs.make_layer(inputs.spec("qwen", T=128, E=4, k=2, H=64, I=64), seed=0)
    out = PT.run_chain(layer)
    assert int(out["status"].item()) == 0
    from oracle import lrmoe_oracle as O
    ref = O.pruned_backward(layer)
    PT.check_selection(layer, out, ref)
    PT.check_gradients(layer, out, ref)


@pytest.mark.parametrize("two_sm", [False, True])
def test_grouped_gemm_stall_times_out_drains_and_context_survives(two_sm):
    """The grouped GEMM itself with its first K block withheld: the MMA issuer's wait
    runs out, the kernel reports LRMOE_ST_TIMEOUT, drains what is in flight, frees
    its tensor memory and returns; the next GEMM on the stream is correct."""
    g = torch.Generator(device="cpu").manual_seed(3)
    E, K, N, rows = 4, 256, 512, 700
    A = torch.randn(rows, K, generator=g).to(torch.bfloat16).cuda()
    W = (0.05 * torch.randn(E, K, N, generator=g)).to(torch.bfloat16).cuda()
    offsets = torch.tensor([0, 200, 420, 420, rows], dtype=torch.int32, device="cuda")
    out = torch.zeros(rows, N, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    L.lrmoe_selftest_gemm_stall(A, W, offsets, out, two_sm, 20000, status)   # 20 ms limit
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(status.item()) & L.ST_TIMEOUT
    assert elapsed < 2.0
    # the same GEMM, run normally right after, is correct
    status.zero_()
    L.lrmoe_grouped_dgrad(A, W, offsets, L.LRMOE_EPI_STORE, out, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    off = offsets.cpu().tolist()
    for e in range(E):
        lo, hi = off[e], off[e + 1]
        if hi == lo:
            continue
        want = A[lo:hi].float() @ W[e].float()
        err = (out[lo:hi].float() - want).norm() / want.norm()
        assert err < 1e-2, (e, float(err))
