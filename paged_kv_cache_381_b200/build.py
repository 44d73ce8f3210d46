"""Build libpa.so in-tree with nvcc for sm_100a.

    python -m paged_kv_cache_381_b200.build [--verbose]

The library holds the CUDA kernels, the C ABI (include/pa.h) and the host
block manager / scheduler (plain C++).  It links the CUDA runtime statically,
so it loads on machines without a GPU (the host-only entry points work there).
"""

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libpa.so")

SOURCES = [
    os.path.join(CSRC, "pa_api.cu"),
    os.path.join(CSRC, "pa_noalloc.cu"),
    os.path.join(CSRC, "host", "block_manager.cpp"),
    os.path.join(CSRC, "host", "scheduler.cpp"),
]

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path():
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _newest_input():
    newest = 0.0
    for d, _, files in os.walk(CSRC):
        for f in files:
            newest = max(newest, os.path.getmtime(os.path.join(d, f)))
    newest = max(newest, os.path.getmtime(os.path.join(ROOT, "include", "pa.h")))
    return newest


def build(verbose=False, force=False, extra_flags=()):
    """Compile libpa.so unless it is newer than every source."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= _newest_input():
        return LIB
    cmd = [nvcc_path(), *ARCH_FLAGS, "-O3", "-lineinfo", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
           "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           *extra_flags, *SOURCES, "-o", LIB + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        print(res.stdout + res.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force=True)
    print(LIB)
