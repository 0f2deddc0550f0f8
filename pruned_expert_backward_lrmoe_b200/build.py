"""Build liblrmoe.so in-tree with nvcc for sm_100a.

    python -m pruned_expert_backward_lrmoe_b200.build [--force] [--verbose] [--checked]

Each csrc/*.cu compiles to _build/<name>.o (in parallel, skipped when newer
than its sources), then everything links into
pruned_expert_backward_lrmoe_b200/liblrmoe.so.  No GPU is needed.

--checked builds the checked-index debug library instead
(pruned_expert_backward_lrmoe_b200/liblrmoe_checked.so, objects under
_build/checked/, compiled with -DLRMOE_CHECKED): every index a kernel takes
from its inputs or its own scans is bounds-checked before use, and one outside
its buffer skips the access and raises LRMOE_ST_BAD_INDEX.  The binding loads
it when LRMOE_CHECKED=1 is set in the environment.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "liblrmoe.so")
LIB_CHECKED = os.path.join(PKG, "liblrmoe_checked.so")
HEADER = os.path.join(ROOT, "include", "lrmoe.h")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "--expt-relaxed-constexpr",
              "-Xptxas", "-O3", "-I" + os.path.join(ROOT, "include")] + ARCH


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps() -> list[str]:
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + [HEADER]


def _compile(src: str, obj: str, verbose: bool, extra: list[str]) -> str:
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-c", src, "-o", obj]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {os.path.basename(src)}:\n{r.stdout}\n{r.stderr}")
    return r.stderr


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False,
          checked: bool = False) -> str:
    bdir = os.path.join(BUILD, "checked") if checked else BUILD
    lib = LIB_CHECKED if checked else LIB
    os.makedirs(bdir, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    dep_time = max(os.path.getmtime(p) for p in _deps())
    jobs = []
    objs = []
    for src in sources:
        obj = os.path.join(bdir, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        fresh = (os.path.exists(obj) and os.path.getmtime(obj) >= os.path.getmtime(src)
                 and os.path.getmtime(obj) >= dep_time)
        if force or not fresh or ptxas_info:
            jobs.append((src, obj))
    extra = (["-Xptxas", "-v"] if ptxas_info else []) + (["-DLRMOE_CHECKED"] if checked else [])
    with cf.ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 4))) as ex:
        futs = {ex.submit(_compile, s, o, verbose, extra): s for s, o in jobs}
        for f in cf.as_completed(futs):
            err = f.result()
            if ptxas_info and err:
                print(f"== {os.path.basename(futs[f])}\n{err}")
    relink = force or bool(jobs) or not os.path.exists(lib) or any(
        os.path.getmtime(o) > os.path.getmtime(lib) for o in objs)
    if relink:
        cmd = [nvcc(), "-shared", *ARCH, "-o", lib, *objs]
        if verbose:
            print(" ".join(cmd), flush=True)
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                ptxas_info="--ptxas-info" in sys.argv, checked="--checked" in sys.argv))
