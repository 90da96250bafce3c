"""Builds libep_b200.so (the CUDA library behind include/ep.h) in-tree, for
sm_100a only.

    python -m combine_ep_get_histogram_b200.build [--force] [--ptxas-verbose]

Floating-point flags: IEEE division and square root, no flush-to-zero, no
automatic FMA contraction (every fused multiply-add in the kernels is an
explicit fmaf), so the results are the ones the kernels spell out.
"""

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libep_b200.so")
SOURCES = ["ep_api.cu", "ep_noalloc.cu", "ep_ipc.cu"]
DEPS = ["common.cuh", "layout.cuh", "movement.cuh", "peers.cuh", "route.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-fmad=false",
    "-Xcompiler", "-fPIC,-O2,-Wall",
    "-shared",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + DEPS] + [os.path.join(INCLUDE, "ep.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if not force and not _stale():
        return LIB
    cmd = [_nvcc()] + NVCC_FLAGS + ["-I", INCLUDE, "-I", CSRC]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-o", LIB + ".tmp"] + [os.path.join(CSRC, f) for f in SOURCES]
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="--ptxas-verbose" in sys.argv))
