"""lrmoe_select_quota_noalloc against lrmoe_select_quota.

The no-allocation entry point is for callers that cannot hand the library any
device scratch: a host framework or plugin host that owns all device memory
and offers its extensions no allocator, or a latency-critical caller that must
not call cudaMalloc/cudaFree because they can synchronise the device.  It uses
a fixed scratch array inside the library instead.  Its outputs are integers, so
the check against the workspace-taking entry point is bit-exact, on calls in a
row with different layers (stale scratch from an earlier call must not leak
into a later one, also when a smaller layer follows a larger one), with the
free device memory unchanged across them, plus the refusal of a problem too
large for the array.

This file is named so that pytest collects it last.
"""
import pytest
import torch

from pruned_expert_backward_lrmoe_b200 import inputs
from pruned_expert_backward_lrmoe_b200 import lrmoe as L

from tests import parity as PT

pytestmark = pytest.mark.gpu


def _scored(spec, seed):
    layer = inputs.make_layer(spec, seed=seed)
    inp = PT.device_inputs(layer)
    s = layer.spec
    score = torch.empty(s.P, dtype=torch.float32, device="cuda")
    L.lrmoe_score(inp["topk_idx"], inp["topk_w"], inp["dY"], inp["a"], s.E, score)
    return layer, inp, score


def _sel_buffers(s):
    i32 = dict(dtype=torch.int32, device="cuda")
    return {"counts": torch.full((s.E,), -7, **i32), "kept": torch.full((s.E,), -7, **i32),
            "offsets": torch.full((s.E + 1,), -7, **i32), "perm": torch.full((s.P,), -7, **i32),
            "pos": torch.full((s.P,), -7, **i32), "status": torch.zeros(1, **i32)}


def _reference(layer, inp, score):
    s = layer.spec
    ref = _sel_buffers(s)
    ws = torch.empty(L.lrmoe_select_workspace_bytes(s.T, s.k, s.E), dtype=torch.uint8, device="cuda")
    L.lrmoe_select_quota(inp["topk_idx"], score, inp["quota"], ref["counts"], ref["kept"],
                         ref["offsets"], ref["perm"], ref["pos"], ws, ref["status"])
    return ref


def _noalloc(layer, inp, score, out=None):
    s = layer.spec
    out = _sel_buffers(s) if out is None else out
    L.lrmoe_select_quota_noalloc(inp["topk_idx"], score, inp["quota"], out["counts"], out["kept"],
                                 out["offsets"], out["perm"], out["pos"], out["status"])
    return out


def _assert_same(got, ref):
    M = int(ref["offsets"][-1].item())
    for name in ("counts", "kept", "offsets", "pos", "status"):
        assert torch.equal(got[name], ref[name]), name
    assert torch.equal(got["perm"][:M], ref["perm"][:M])


def test_noalloc_selection_matches_workspace_selection_twice():
    a = _scored(inputs.spec("skew", T=2048, E=16, k=4, H=128, I=128), seed=0)
    b = _scored(inputs.spec("qwen", T=4096, E=64, k=8, H=64, I=64), seed=1)
    ref_a = _reference(*a)
    ref_b = _reference(*b)
    # every output buffer exists before the no-alloc calls, so that the free
    # device memory measured around them can only change if they allocate
    outs = [_sel_buffers(a[0].spec), _sel_buffers(b[0].spec), _sel_buffers(a[0].spec)]
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    got_a = _noalloc(*a, out=outs[0])   # first call: also looks up the scratch address
    got_b = _noalloc(*b, out=outs[1])   # second call in a row reuses the same scratch
    # third call: the smaller layer again, after the larger one left its bytes
    # beyond the smaller layout in the shared array
    got_a2 = _noalloc(*a, out=outs[2])
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    _assert_same(got_a, ref_a)
    _assert_same(got_b, ref_b)
    _assert_same(got_a2, ref_a)
    assert int(ref_b["offsets"][-1].item()) > 0
    assert free_after == free_before, (free_before, free_after)


def test_noalloc_refuses_problems_larger_than_its_array():
    T, k, E = 131072, 8, 128                   # 1 M pairs: needs ~8 MiB of scratch
    assert L.lrmoe_select_workspace_bytes(T, k, E) > L.NOALLOC_SCRATCH_BYTES
    i32 = dict(dtype=torch.int32, device="cuda")
    idx = torch.zeros(T, k, **i32)
    score = torch.zeros(T * k, dtype=torch.float32, device="cuda")
    quota = torch.zeros(E, **i32)
    outs = [torch.full((n,), -7, **i32) for n in (E, E, E + 1, T * k, T * k)]
    with pytest.raises(L.LrmoeError) as err:
        L.lrmoe_select_quota_noalloc(idx, score, quota, *outs)
    assert err.value.code == L.LRMOE_ERR_WORKSPACE
    assert "built-in" in str(err.value)
    torch.cuda.synchronize()
    assert all(bool((o == -7).all()) for o in outs)   # nothing was written
