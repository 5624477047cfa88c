"""Build libpoem.so (the CUDA library behind include/poem.h) in-tree for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libpoem.so")
SOURCES = ["poem_api.cu", "bsa_fwd.cu", "bsa_fwd_grouped.cu", "poem_score.cu", "poem_select.cu", "poem_select_noalloc.cu", "poem_pooled.cu"]
HEADERS = ["sm100.cuh", "common.cuh", "fwd_common.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr", "-I" + os.path.join(ROOT, "include"),
]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(ROOT, "include", "poem.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or _stale():
        cmd = [NVCC, *FLAGS]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        cmd += ["-o", LIB] + [os.path.join(CSRC, f) for f in SOURCES]
        subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="-v" in sys.argv)
    print(LIB)
