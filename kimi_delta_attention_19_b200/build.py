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


def _compile(src: str, obj: str, extra: list[str] | None = None) -> str:
    cmd = [_nvcc(), *ARCH, *NVCC_FLAGS, *(extra or []), "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return r.stderr  # ptxas -v report


# Test-only variant of the library: the first wait on the inputs in each tensor-core prefill
# kernel gives up after 64 clocks, so a test can watch the kernels' bail-out path (status
# word set, copies and products drained, tensor memory freed) run on the GPU and the
# context stay usable. The product never loads it.
SHORTWAIT_LIB = os.path.join(PKG, "libkda_shortwait.so")
SHORTWAIT_DEFINES = {"kda_prefill_tc.cu": ["-DKDA_FIRST_WAIT_LIMIT=64", "-DKDA_FIRST_WAIT_STUCK=1"]}


def _link(lib: str, objs: list[str]) -> None:
    if os.path.exists(lib) and os.path.getmtime(lib) >= max(os.path.getmtime(o) for o in objs):
        return
    cmd = [_nvcc(), *ARCH, "-shared", "-cudart", "static", "-o", lib, *objs]
    subprocess.run(cmd, check=True)


def build(verbose: bool = False) -> str:
    os.makedirs(BUILD, exist_ok=True)
    sources = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    deps = sources + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        [os.path.join(ROOT, "include", "kda.h")]
    newest_dep = max(os.path.getmtime(p) for p in deps)
    objs, short_objs = [], []
    jobs = {}
    with cf.ThreadPoolExecutor(max_workers=min(8, len(sources) + len(SHORTWAIT_DEFINES))) as ex:
        for src in sources:
            name = os.path.basename(src)
            obj = os.path.join(BUILD, name + ".o")
            objs.append(obj)
            todo = [(obj, [])]
            if name in SHORTWAIT_DEFINES:
                sobj = os.path.join(BUILD, name + ".shortwait.o")
                short_objs.append(sobj)
                todo.append((sobj, SHORTWAIT_DEFINES[name]))
            else:
                short_objs.append(obj)
            for o, extra in todo:
                if os.path.exists(o) and os.path.getmtime(o) >= newest_dep:
                    continue
                jobs[ex.submit(_compile, src, o, extra)] = (name, extra)
        for fut in cf.as_completed(jobs):
            report = fut.result()
            if verbose:
                print(f"== {jobs[fut][0]} {' '.join(jobs[fut][1])}\n{report}", file=sys.stderr)
    _link(LIB, objs)
    _link(SHORTWAIT_LIB, short_objs)
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv))
