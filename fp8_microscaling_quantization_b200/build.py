"""Build libbsq.so in-tree with nvcc for sm_100a.

    python -m fp8_microscaling_quantization_b200.build [--force] [--debug]

Flags: -gencode arch=compute_100a,code=sm_100a, -O3, -lineinfo, no fast-math
(IEEE division, denormals kept), -fmad=false (no multiply-add contraction, so
the binary32 scale arithmetic rounds exactly where the formulas round).  The
CUDA runtime is linked statically and the driver entry point for tensor maps
is resolved at run time, so the library loads on a machine without a GPU.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libbsq.so")
# the bounds-checking build (-DBSQ_DEBUG): every checked index is tested
# against its extent, a failure is counted, not trapped (csrc/debug.cuh)
LIB_DEBUG = os.path.join(HERE, "libbsq_debug.so")
SOURCES = ["abi.cu", "flat.cu", "nvfp4.cu", "static.cu", "kv_cache.cu", "cache.cu", "grouped_mm.cu"]
HEADERS = ["common.cuh", "formats.cuh", "host_util.h", "tcgen05.cuh", "debug.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-fmad=false", "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-Xptxas", "-warn-spills",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES]
    files += [os.path.join(CSRC, h) for h in HEADERS if os.path.exists(os.path.join(CSRC, h))]
    files.append(os.path.join(ROOT, "include", "bsq.h"))
    return files


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def _wait_all(procs):
    failed = [p.args for p in procs if p.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, failed[0])


def build(force: bool = False, verbose: bool = False, extra_flags=None, debug: bool = False) -> str:
    """Compile every source (in parallel, one nvcc per file) and link;
    debug=True builds the bounds-checking libbsq_debug.so instead."""
    lib = LIB_DEBUG if debug else LIB
    if debug:
        extra_flags = list(extra_flags or []) + ["-DBSQ_DEBUG"]
    if not force and up_to_date(lib):
        return lib
    objs, cmds = [], []
    tag = "dbg." if debug else ""
    for src in SOURCES:
        obj = os.path.join(CSRC, src.replace(".cu", f".{tag}{os.getpid()}.o"))
        cmds.append([nvcc(), *NVCC_FLAGS, *(extra_flags or []), "-I", os.path.join(ROOT, "include"), "-c",
                     os.path.join(CSRC, src), "-o", obj])
        objs.append(obj)
    jobs = max(1, min(len(cmds), os.cpu_count() or 1))
    running = []
    for cmd in cmds:
        if verbose:
            print(" ".join(cmd), flush=True)
        running.append(subprocess.Popen(cmd))
        if len(running) >= jobs:
            _wait_all(running[:1])
            running = running[1:]
    _wait_all(running)
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-Xcompiler", "-fPIC", *objs, "-o", tmp]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    for o in objs:
        os.remove(o)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv)
