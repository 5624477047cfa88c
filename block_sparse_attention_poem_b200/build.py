"""Build libpoem.so (the CUDA library behind include/poem.h) in-tree for sm_100a.

variant="checks" builds libpoem_checks.so, the same sources compiled with
-DPOEM_CHECKS: device-side bounds checks that skip an out-of-range access and
report POEM_ERR_BOUNDS through poem_check.  The binding loads it when the
environment variable POEM_LIBRARY_VARIANT is "checks"."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libpoem.so")
LIBS = {"release": LIB, "checks": os.path.join(PKG, "libpoem_checks.so")}
SOURCES = ["poem_api.cu", "bsa_fwd.cu", "bsa_fwd_grouped.cu", "poem_score.cu", "poem_score_pass1.cu", "poem_select.cu", "poem_select_noalloc.cu", "poem_pooled.cu"]
HEADERS = ["sm100.cuh", "common.cuh", "fwd_common.cuh", "score_common.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr", "-I" + os.path.join(ROOT, "include"),
]


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(ROOT, "include", "poem.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, variant: str = "release") -> str:
    lib = LIBS[variant]
    if force or _stale(lib):
        cmd = [NVCC, *FLAGS]
        if variant == "checks":
            cmd += ["-DPOEM_CHECKS"]
        if verbose:
            cmd += ["-Xptxas", "-v"]
        cmd += ["-o", lib] + [os.path.join(CSRC, f) for f in SOURCES]
        subprocess.run(cmd, check=True)
    return lib


if __name__ == "__main__":
    v = "checks" if "--checks" in sys.argv else "release"
    print(build(force=True, verbose="-v" in sys.argv, variant=v))
