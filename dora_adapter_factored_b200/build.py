"""Builds libdora.so in-tree with nvcc for sm_100a (B200).

Usage:  python -m dora_adapter_factored_b200.build [--verbose]
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libdora.so"

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared",
    "-cudart", "static",
    "--expt-relaxed-constexpr",
]


DEBUG_LIB_NAME = "libdora_debug.so"


def library_path(debug: bool = False) -> str:
    """The in-tree library; `debug`: the DORA_DEBUG build, whose kernels check
    the index of every computed-address global store, skip an out-of-range one
    and record DORA_ERR_BOUNDS in the device status word."""
    return os.path.join(PKG, DEBUG_LIB_NAME if debug else LIB_NAME)


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def is_stale(debug: bool = False) -> bool:
    lib = library_path(debug)
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in _sources())


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libdora.so")


def build(verbose: bool = False, extra_flags=(), debug: bool = False) -> str:
    out = library_path(debug)
    tmp = out + ".tmp"
    if debug:
        extra_flags = [*extra_flags, "-DDORA_DEBUG"]
    cmd = [nvcc(), *NVCC_FLAGS, *extra_flags, "-I", INCLUDE, "-I", CSRC,
           os.path.join(CSRC, "dora.cu"), "-o", tmp]
    if verbose:
        print(" ".join(cmd))
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose and (res.stdout or res.stderr):
        print(res.stdout, res.stderr)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv,
                extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [],
                debug="--debug" in sys.argv))
