"""Builds librz.so (the C ABI of include/rz.h) in-tree with nvcc for sm_100a only."""
from __future__ import annotations

import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "librz.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [os.path.join(ROOT, "include", "rz.h")]


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in deps())


def build(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    """Compile every .cu under csrc/ into librz.so (nvcc, -gencode arch=compute_100a,code=sm_100a)."""
    if not force and not needs_build():
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, *NVCC_FLAGS, *extra_flags, "-I", os.path.join(ROOT, "include"), *sources(), "-o", LIB + ".tmp"]
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


def source_digest(family: str = "all") -> str:
    """sha256 prefix over the sources that define a kernel family.

    "gemm": the tensor-core engine, its epilogues and the launch code; "simt": the
    SIMT kernels and the launch code; "all": every CUDA source and the public header.
    A recorded measurement of a kernel is only current while its family's digest holds.
    """
    import hashlib
    names = {
        "gemm": ("rz_ptx.cuh", "rz_gemm.cuh", "rz_epilogues.cuh", "rz_api.cu"),
        "simt": ("rz_ptx.cuh", "rz_epilogues.cuh", "rz_simt.cuh", "rz_api.cu"),
    }
    paths = deps() if family == "all" else [os.path.join(CSRC, n) for n in names[family]]
    h = hashlib.sha256()
    for p in paths:
        h.update(os.path.basename(p).encode())
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


if __name__ == "__main__":
    import sys
    build(force="--force" in sys.argv, verbose=True,
          extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
