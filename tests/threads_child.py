"""Child process of test_threads_gpu.py: the library's first calls in a fresh
process come from four host threads at once.

Each thread owns a stream and its buffers and runs the whole path
(lrmoe_pruned_backward: score, selection, compaction, grouped GEMMs, unpack)
on one of two bf16 layers; the threads are released together by a barrier, so
the one-time host set-up inside the library (tensor-map encoder lookup, kernel
attributes, SM count) is reached concurrently.  Every thread's result is then
checked against the CPU oracle.  Prints "threads ok" and exits 0 on success.
"""
from __future__ import annotations

import os
import sys
import threading

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main() -> int:
    import torch

    from oracle import lrmoe_oracle as O
    from pruned_expert_backward_lrmoe_b200 import inputs
    from pruned_expert_backward_lrmoe_b200 import lrmoe as L
    from tests import parity as PT

    specs = [inputs.spec("qwen", T=512, E=8, k=4, H=256, I=192),
             inputs.spec("qwen", T=300, E=6, k=3, H=320, I=136, quota="half_ceil")]
    layers = [inputs.make_layer(s, seed=0) for s in specs]
    refs = [O.pruned_backward(layer) for layer in layers]
    torch.cuda.set_device(0)
    n_threads = 4
    jobs = []
    for i in range(n_threads):
        layer = layers[i % 2]
        s = layer.spec
        inp = PT.device_inputs(layer)
        out = L.alloc_buffers(s.T, s.k, s.E, s.H, s.I, torch.bfloat16)
        out["status"].zero_()
        jobs.append((layer, inp, out, torch.cuda.Stream()))
    torch.cuda.synchronize()
    gate = threading.Barrier(n_threads)
    errors = []

    def work(i):
        layer, inp, out, stream = jobs[i]
        try:
            torch.cuda.set_device(0)
            gate.wait()
            L.lrmoe_pruned_backward(inp, out, stream=stream)
        except Exception as exc:  # reported by the main thread
            errors.append(f"thread {i}: {exc!r}")

    threads = [threading.Thread(target=work, args=(i,)) for i in range(n_threads)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    torch.cuda.synchronize()
    if errors:
        print("\n".join(errors))
        return 1
    for i, (layer, _, out, _) in enumerate(jobs):
        ref = refs[i % 2]
        M = PT.check_selection(layer, out, ref)
        PT.check_pack(layer, out, ref, M, PT.chain_packed(layer))
        PT.check_gradients(layer, out, ref)
        assert int(out["status"].item()) == 0, f"thread {i}: device status {int(out['status'].item())}"
    print("threads ok")
    return 0


if __name__ == "__main__":
    sys.exit(main())
