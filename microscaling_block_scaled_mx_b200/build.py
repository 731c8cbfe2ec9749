"""Build libmx.so (the C-ABI library) in-tree with nvcc for sm_100a, and on
request libmx_debug.so: the same sources compiled with MX_DEBUG, whose cast
kernels (MX, dual and NVFP4) check every code and scale store, and the
decode its loads, against the buffer sizes, and report a range outside a
buffer as MX_ERR_BOUNDS instead of touching it.

Usage: python -m microscaling_block_scaled_mx_b200.build [--force] [--debug]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libmx.so")
DEBUG_LIB = os.path.join(PKG, "libmx_debug.so")
SOURCES = ["mx_api.cu", "mx_cast.cu", "mx_gemm.cu", "mx_nvfp4.cu"]

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    # bit-exact arithmetic: IEEE division/sqrt, no flush-to-zero, no FMA contraction
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-fmad=false",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "mx.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = DEBUG_LIB if debug else LIB
    if not force and not _stale(lib):
        return lib
    tmp_dir = os.path.join(PKG, "_build_debug" if debug else "_build")
    os.makedirs(tmp_dir, exist_ok=True)
    jobs = []
    for src in SOURCES:
        obj = os.path.join(tmp_dir, src.replace(".cu", ".o"))
        cmd = [nvcc(), *NVCC_FLAGS, *(["-DMX_DEBUG"] if debug else []), "-I", INCLUDE, "-I", CSRC, "-c",
               os.path.join(CSRC, src), "-o", obj]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), flush=True)
        jobs.append((obj, cmd))
    # the translation units are independent: compile them concurrently
    procs = [(obj, cmd, subprocess.Popen(cmd)) for obj, cmd in jobs]
    failed = [cmd for _, cmd, proc in procs if proc.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, failed[0])
    objs = [obj for obj, _ in jobs]
    tmp_lib = lib + f".tmp{os.getpid()}"
    subprocess.run([nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp_lib, *objs,
                    "-lcudart"], check=True)
    os.replace(tmp_lib, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
