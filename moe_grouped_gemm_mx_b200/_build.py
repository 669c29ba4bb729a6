"""Ahead-of-time build of the sm_100a library ``libmx.so`` (no JIT).

    python moe_grouped_gemm_mx_b200/_build.py          # build if stale
    python moe_grouped_gemm_mx_b200/_build.py --force  # rebuild

(run as a file, not as a package module: importing the package loads the
library, which is what this script builds)

nvcc cross-compiles for sm_100a on a machine without a GPU, so the library is
built in-tree and travels with the source tree.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libmx.so")
SOURCES = ["mx_api.cu", "mx_gemm.cu", "mx_gemm2.cu", "mx_quant.cu", "mx_quant_t.cu", "mx_quant_tw.cu",
           "mx_gemm_tw.cu", "mx_moe.cu"]
HEADERS = ["mx_ptx.cuh", "mx_launch.h", "mx_fastdiv.h", "mx_gemm_common.cuh", "mx_mxfp8.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "mx.h"))
    files.append(os.path.abspath(__file__))
    return files


def is_stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    if not force and not is_stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc_path(), *ARCH, "-lineinfo", "-O3", "-std=c++17", "--shared", "-Xcompiler", "-fPIC",
           "-I", os.path.join(ROOT, "include"), "-o", tmp]
    if ptxas_info:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, ptxas_info="-v" in sys.argv)
    print(LIB)
