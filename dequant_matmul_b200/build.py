"""Builds libhlwq.so in-tree with nvcc for sm_100a (no GPU needed)."""

from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libhlwq.so")
# The same sources with the failure-detection hooks compiled in (tests only).
FAULT_LIB = os.path.join(PKG, "libhlwq_fault.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "--expt-relaxed-constexpr", "--extended-lambda",
    "-Xcompiler", "-fPIC,-O3",
    "-shared",
]


def sources():
    return [os.path.join(PKG, "csrc", "libhlwq.cu"), os.path.join(PKG, "csrc", "noalloc.cu"),
            os.path.join(PKG, "csrc", "codebook.cpp")]


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + glob.glob(os.path.join(PKG, "csrc", "*.cuh")) + glob.glob(os.path.join(ROOT, "include", "*.h"))
    return any(os.path.getmtime(p) > t for p in deps)


def build(verbose: bool = False, force: bool = False, extra=None) -> str:
    """Builds libhlwq.so and libhlwq_fault.so (two nvcc runs in parallel)."""
    nvcc = os.environ.get("NVCC", "nvcc")
    jobs = []
    for lib, defs in ((LIB, []), (FAULT_LIB, ["-DHLWQ_FAULT_INJECTION"])):
        if not force and not needs_build(lib):
            continue
        cmd = [nvcc, *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), *defs, *(extra or []), "-o", lib + ".tmp",
               *sources()]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        jobs.append((lib, subprocess.Popen(cmd)))
    failed = [lib for lib, p in jobs if p.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, f"nvcc ({', '.join(os.path.basename(f) for f in failed)})")
    for lib, _ in jobs:
        os.replace(lib + ".tmp", lib)
    return LIB


if __name__ == "__main__":
    build(verbose=True, force="--force" in sys.argv,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
