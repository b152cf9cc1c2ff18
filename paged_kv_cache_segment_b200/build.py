"""Build libtfpaged.so in this package directory with nvcc for sm_100a.

    python -m paged_kv_cache_segment_b200.build [--verbose-ptxas]

The shared library exports exactly the C ABI of include/tfpaged.h.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libtfpaged.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared",
         "--expt-relaxed-constexpr", "-Wno-deprecated-gpu-targets"]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def headers() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(HERE, "..", "include", "tfpaged.h")])


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in sources() + headers())


def build(verbose_ptxas: bool = False, force: bool = False) -> str:
    if not force and not stale():
        return LIB
    cmd = [NVCC, *ARCH, *FLAGS, "-I", os.path.join(HERE, "..", "include"), *sources(), "-o", LIB]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(verbose_ptxas="--verbose-ptxas" in sys.argv, force=True)
    print(LIB)
