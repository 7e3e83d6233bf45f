"""Build the CUDA library libgm_b200.so (sm_100a) next to this file.

    python -m sparse_dynamic_routing_b200.build [--force] [--verbose]

One translation unit (csrc/gm_api.cu) with the C ABI of include/gm.h (--checked builds the
variant that verifies every input edge tensor, libgm_b200_checked.so); the CUDA runtime is
linked statically, so the library only needs the NVIDIA driver at run time. No fast-math:
the referral step relies on IEEE fp32 products and sums (it uses the _rn intrinsics), and
denormals are kept (-ftz=false).
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libgm_b200.so")
# the checked build: every call first verifies the edge tensors it reads (GM_CHECKED=1)
CHECKED_LIB = os.path.join(HERE, "libgm_b200_checked.so")
HEADER = os.path.join(ROOT, "include", "gm.h")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-ftz=false", "-prec-div=true", "-prec-sqrt=true",
    "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [HEADER])


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    lib = CHECKED_LIB if checked else LIB
    if force or stale(lib):
        tmp = lib + f".tmp{os.getpid()}"
        cmd = [nvcc(), *NVCC_FLAGS, *(["-DGM_CHECKED=1"] if checked else []),
               os.path.join(CSRC, "gm_api.cu"), "-o", tmp]
        if verbose:
            cmd[1:1] = ["-Xptxas", "-v"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv,
                checked="--checked" in sys.argv))
