"""Build libmacaq.so (sm_100a) in-tree with nvcc.

    python -m online_hadamard_b200.build        # or online_hadamard_b200.build.build()

The library is one translation unit (csrc/libmacaq.cu); the output goes to
online_hadamard_b200/_build/libmacaq.so next to the sources, so it travels with the tree.
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
INCLUDE = os.path.join(ROOT, "include")
BUILD_DIR = os.path.join(HERE, "_build")
LIB_PATH = os.path.join(BUILD_DIR, "libmacaq.so")
# Fault-injection build for the tests only: stream-K owners give up on a flag after 200 000 cycles
# (~0.1 ms) instead of ~4 s, and macaq_test_owner_tag_offset() can make them wait for a tag that no
# contributor writes, so a test can see a bounded device-side wait run out.  Never loaded by the
# product path.
FAULT_LIB_PATH = os.path.join(BUILD_DIR, "libmacaq_faultwait.so")
FAULT_FLAGS = ["-DMACAQ_TEST_HOOKS", "-DMACAQ_FLAG_WAIT_LIMIT=200000"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; the CUDA toolkit is required to build libmacaq")
    return cand


def _sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(INCLUDE, "macaq.h")])


def is_stale(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return True
    t = os.path.getmtime(path)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, verbose: bool = False, extra_flags: list[str] | None = None,
          path: str = LIB_PATH) -> str:
    if not force and not is_stale(path):
        return path
    os.makedirs(BUILD_DIR, exist_ok=True)
    tmp = path + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, *(extra_flags or []), "-I", INCLUDE, "-I", CSRC,
           "-o", tmp, os.path.join(CSRC, "libmacaq.cu")]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, path)
    return path


def build_fault_library(force: bool = False) -> str:
    """The fault-injection build (tests only), next to the product library."""
    return build(force=force, extra_flags=FAULT_FLAGS, path=FAULT_LIB_PATH)


if __name__ == "__main__":
    v = "-v" in sys.argv
    flags = ["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None
    print(build(force=True, verbose=v, extra_flags=flags))
    print(build_fault_library(force=True))
