"""Build libac.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

    python -m cluster_routed_sparse_b200.build [--verbose-ptxas]
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libac.so")
SOURCES = ["ac_api.cu", "cluster_kernels.cu", "assign_mma.cu", "score_kernels.cu", "quest_mma.cu", "attn_kernel.cu",
           "noalloc.cu"]
HEADERS = ["ac_device.cuh", "ac_internal.h"]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for p in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if p and (os.path.isabs(p) and os.path.exists(p) or not os.path.isabs(p)):
            return p
    return "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "ac.h")]
    return any(os.path.getmtime(f) > t for f in deps)


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    """Compile every CUDA source into one shared library next to this file."""
    if not force and not _stale():
        return LIB
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-I", INCLUDE, "-I", CSRC,
           "-o", LIB + ".tmp"] + [os.path.join(CSRC, f) for f in SOURCES] + ["-lcudart"]
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)
