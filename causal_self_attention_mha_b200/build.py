"""Builds libcausalattn.so in-tree with nvcc for sm_100a (B200).

The library is one translation unit (csrc/causalattn.cu) that includes the
kernel headers; it links the CUDA runtime statically, so the only runtime
dependency is the NVIDIA driver.  `build(debug=True)` builds the same sources
with CA_DEBUG_CHECKS into libcausalattn_debug.so: the kernels then check every
TMA coordinate and computed global index on the device and record a failed
check in the device status word instead of making the access.
"""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libcausalattn.so")
LIB_DEBUG = os.path.join(HERE, "libcausalattn_debug.so")
ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + glob.glob(os.path.join(ROOT, "include", "*.h")))


def is_stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def nvcc_command(out: str, debug: bool = False, verbose: bool = False):
    cmd = [nvcc_path(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
           "-shared", "-cudart", "static", "-I", os.path.join(ROOT, "include"),
           "-o", out, os.path.join(CSRC, "causalattn.cu")]
    if debug:
        cmd.insert(1, "-DCA_DEBUG_CHECKS")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and not is_stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.run(nvcc_command(tmp, debug, verbose), check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                debug="--debug" in sys.argv))
