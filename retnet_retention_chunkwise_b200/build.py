"""Build libretention.so in-tree with nvcc for sm_100a.

The library is one translation unit (csrc/retention_abi.cu includes every
kernel).  The CUDA runtime is linked statically, so the .so only needs the
driver at run time; the tensor-map encoder is fetched from the driver through
cudaGetDriverEntryPoint.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libretention.so")
# The same library with index checks in the kernels (-DRET_BOUNDS_CHECK): a
# failed check skips its access and the device status reads RET_EBOUNDS.  For
# tests only; select it with RETENTION_LIBRARY=<path>.
LIB_BOUNDS_CHECK = os.path.join(HERE, "libretention_bc.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cu", ".cuh"))] + [
        os.path.join(os.path.dirname(HERE), "include", "retention.h")]


def stale(out: str = LIB) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(s) > t for s in sources())


def build(out: str = LIB, extra=(), verbose: bool = False) -> str:
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr", "-cudart", "static",
           *extra, os.path.join(CSRC, "retention_abi.cu"), "-o", out]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    return out


def build_bounds_check(out: str = LIB_BOUNDS_CHECK, verbose: bool = False) -> str:
    return build(out, extra=("-DRET_BOUNDS_CHECK",), verbose=verbose)


if __name__ == "__main__":
    build(verbose="-v" in sys.argv)
    print(LIB)
    if "--bounds-check" in sys.argv:
        build_bounds_check()
        print(LIB_BOUNDS_CHECK)
