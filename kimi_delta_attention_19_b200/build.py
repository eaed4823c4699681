"""Build libkda.so (the C-ABI CUDA library) in-tree for sm_100a.

    python -m kimi_delta_attention_19_b200.build

Each .cu under csrc/ is compiled by nvcc in parallel into _build/, then linked
into kimi_delta_attention_19_b200/libkda.so. Nothing is JIT-compiled at import.
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
LIB = os.path.join(PKG, "libkda.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
              "--expt-relaxed-constexpr", "-Xptxas", "-v", "-I", os.path.join(ROOT, "include")]


def _nvcc() -> str:
    cuda_home = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    p = os.path.join(cuda_home, "bin", "nvcc")
    return p if os.path.exists(p) else (shutil.which("nvcc") or "nvcc")


def _compile(src: str, obj: str) -> str:
    cmd = [_nvcc(), *ARCH, *NVCC_FLAGS, "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return r.stderr  # ptxas -v report


def build(verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    deps = sources + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        [os.path.join(ROOT, "include", "kda.h")]
    newest_dep = max(os.path.getmtime(p) for p in deps)
    objs = []
    jobs = {}
    with cf.ThreadPoolExecutor(max_workers=min(8, len(sources))) as ex:
        for src in sources:
            obj = os.path.join(BUILD, os.path.basename(src) + ".o")
            objs.append(obj)
            if os.path.exists(obj) and os.path.getmtime(obj) >= newest_dep:
                continue
            jobs[ex.submit(_compile, src, obj)] = src
        for fut in cf.as_completed(jobs):
            report = fut.result()
            if verbose:
                print(f"== {os.path.basename(jobs[fut])}\n{report}", file=sys.stderr)
    if (not os.path.exists(LIB) or jobs
            or os.path.getmtime(LIB) < max(os.path.getmtime(o) for o in objs)):
        cmd = [_nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", LIB, *objs]
        subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
