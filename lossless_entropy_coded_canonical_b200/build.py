"""Builds libdfw.so in-tree with nvcc for sm_100a (B200).

``python -m lossless_entropy_coded_canonical_b200.build`` or :func:`build`.
The host half (encoder, planner) and the device half (kernels) go into one
shared library; the CUDA runtime is linked statically so the library shares
the driver's primary context with whatever framework loaded it.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libdfw.so")
# the checks build: every copy range, shared-memory extent and output index
# the kernels compute is checked before use (DFW_CHECKS)
LIB_CHECKS = os.path.join(PKG, "libdfw_checks.so")
SOURCES = ["dfw_host.cpp", "dfw_decode.cu", "dfw_encode.cu", "dfw_rans.cpp"]
HEADERS = ["dfw_internal.h", "dfw_device.cuh", "dfw_lanes.cuh", "dfw_rans.cuh", os.path.join("..", "..", "include", "dfw.h")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found; libdfw needs the CUDA toolkit to build")


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.abspath(__file__)]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, checks: bool = False) -> str:
    """Builds libdfw.so (or, with checks, libdfw_checks.so) unless it is newer
    than every source."""
    lib = LIB_CHECKS if checks else LIB
    if not force and not _stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3,-pthread",
           *(["-DDFW_CHECKS"] if checks else []), "-shared", "-o", tmp, *[os.path.join(CSRC, f) for f in SOURCES]]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, checks="--checks" in sys.argv))
