"""Build libmx.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: python -m microscaling_block_scaled_mx_b200.build [--force]
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


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, "mx.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    tmp_dir = os.path.join(PKG, "_build")
    os.makedirs(tmp_dir, exist_ok=True)
    jobs = []
    for src in SOURCES:
        obj = os.path.join(tmp_dir, src.replace(".cu", ".o"))
        cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, "-c", os.path.join(CSRC, src), "-o", obj]
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
    tmp_lib = LIB + f".tmp{os.getpid()}"
    subprocess.run([nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", tmp_lib, *objs,
                    "-lcudart"], check=True)
    os.replace(tmp_lib, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
