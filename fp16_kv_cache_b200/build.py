"""Build libhyq.so in-tree from csrc/*.cu for sm_100a (B200).

    python -m fp16_kv_cache_b200.build [--force] [--verbose]

nvcc cross-compiles without a GPU; the shared object lands next to this file
so it travels with the source tree.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libhyq.so")
# The same sources built with -DHYQ_DEBUG: device-side index checks that
# raise HYQ_DEV_OOB, and a host-settable limit for the decode's bounded
# waits (hyq_debug_set_wait_limit, include/hyq_debug.h).  For tests.
DEBUG_LIB = os.path.join(HERE, "libhyq_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _inputs())


def _compile(lib: str, defines=(), verbose: bool = False) -> str:
    cmd = [
        NVCC, "-O3", "-std=c++17",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
        "-I", INCLUDE,
        "-o", lib + ".tmp",
    ] + [f"-D{d}" for d in defines] + sources()
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd, cwd=CSRC)
    os.replace(lib + ".tmp", lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    """Build libhyq.so (and, unless HYQ_SKIP_DEBUG_LIB is set, the debug
    library beside it) when a source is newer than the library."""
    if force or needs_build(LIB):
        _compile(LIB, verbose=verbose)
    if not os.environ.get("HYQ_SKIP_DEBUG_LIB"):
        build_debug(force)
    return LIB


def build_debug(force: bool = False) -> str:
    if force or needs_build(DEBUG_LIB):
        _compile(DEBUG_LIB, defines=("HYQ_DEBUG",))
    return DEBUG_LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
