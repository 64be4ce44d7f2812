"""Build libint8lt.so in-tree with nvcc for sm_100a (no GPU needed to build).

Two libraries from the same sources: libint8lt.so, and libint8lt_check.so,
compiled with -DINT8LT_DEBUG, whose kernels check the index of their computed
global accesses and report a failed check as INT8LT_ERR_BOUNDS (device
status) instead of making the access.
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
SOURCES = ["api.cu", "quantize.cu", "gemm_tc.cu", "gemv.cu", "static_scratch.cu",
           "zeropoint.cu", "weight_layout.cu"]
LIB = os.path.join(HERE, "libint8lt.so")
CHECK_LIB = os.path.join(HERE, "libint8lt_check.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
         "-Xcompiler", "-fPIC"]


def _stale(out: str, deps: list[str]) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def _link(objs: list[str], out: str) -> None:
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                           "-o", tmp, *objs])
    os.replace(tmp, out)


def build(force: bool = False, verbose: bool = False) -> str:
    """Build both libraries if any source is newer; returns the regular one's path."""
    deps = [os.path.join(CSRC, s) for s in SOURCES]
    deps += [os.path.join(CSRC, "int8lt_internal.cuh"),
             os.path.join(HERE, "..", "include", "int8lt.h")]
    todo = [(out, extra) for out, extra in ((LIB, []), (CHECK_LIB, ["-DINT8LT_DEBUG"]))
            if force or _stale(out, deps)]
    if not todo:
        return LIB
    objdir = os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    jobs = []
    for out, extra in todo:
        tag = "check_" if extra else ""
        for src in SOURCES:
            obj = os.path.join(objdir, tag + src.replace(".cu", ".o"))
            cmd = [NVCC, *FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
            if verbose:
                cmd += ["-Xptxas", "-v"]
            jobs.append((out, obj, cmd))
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as pool:
        for f in [pool.submit(subprocess.check_call, cmd) for _, _, cmd in jobs]:
            f.result()
    for out, _ in todo:
        _link([obj for o, obj, _ in jobs if o == out], out)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
