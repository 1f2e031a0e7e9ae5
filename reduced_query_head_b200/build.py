"""Build libsqa.so in-tree for sm_100a (nvcc; no GPU needed to compile)."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libsqa.so")
# Debug build: the same library with device bounds checks (SQA_DEBUG_BOUNDS) that
# record SQA_ERR_BOUNDS in the device status word instead of faulting.
LIB_DEBUG = os.path.join(HERE, "libsqa_debug.so")
SOURCES = ["sqa.cu"]
HEADERS = ["sm100.cuh", "attn_fwd.cuh", "attn_bwd.cuh", "decode.cuh", "gemm.cuh"]
INCLUDE = os.path.join(ROOT, "include")

NVCC_FLAGS = [
    "-O3", "-std=c++17",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo",
    "-Xcompiler", "-fPIC",
    "-shared",
]


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "sqa.h"))
    files.append(os.path.abspath(__file__))
    return files


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and not needs_build(lib):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = lib + ".tmp%d" % os.getpid()
    flags = NVCC_FLAGS + (["-DSQA_DEBUG_BOUNDS"] if debug else [])
    cmd = [nvcc, *flags, "-I", INCLUDE, "-o", tmp] + [os.path.join(CSRC, f) for f in SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv)
    print(LIB_DEBUG if "--debug" in sys.argv else LIB)
