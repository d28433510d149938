"""Build the DF11 CUDA library in-tree for sm_100a (nvcc, static CUDA runtime)."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libdf11_b200.so")
# The same sources with test hooks (not the product): a decode whose bounded
# waits are made to run out, and a short wait limit so that they do quickly.
TEST_LIB = os.path.join(HERE, "libdf11_b200_test.so")
TEST_FLAGS = ["-DDF11_TEST_HOOKS", "-DDF11_WAIT_LIMIT=256u"]
# The checked build: bounds checks on every shared-memory access and global
# store of the decode path, reported as DF11_ERR_BOUNDS instead of a fault.
CHECKED_LIB = os.path.join(HERE, "libdf11_b200_checked.so")
CHECKED_FLAGS = ["-DDF11_CHECKED"]
SOURCES = [os.path.join(CSRC, "df11_kernels.cu"), os.path.join(CSRC, "df11_host.cpp"),
           os.path.join(CSRC, "rans_kernels.cu"), os.path.join(CSRC, "rans_host.cpp")]
HEADERS = [os.path.join(CSRC, "df11_internal.h"), os.path.join(CSRC, "df11_codebook.h"),
           os.path.join(INCLUDE, "df11.h"), os.path.join(INCLUDE, "df11_rans.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2,-Wall",
    "-Xptxas", "-v",
    "-shared", "-cudart", "static",
]


def _stale(lib: str) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in SOURCES + HEADERS)


def _nvcc(lib: str, extra, verbose: bool) -> str:
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC, *SOURCES, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    """The product library, libdf11_b200.so."""
    if not force and not _stale(LIB):
        return LIB
    return _nvcc(LIB, [], verbose)


def build_test(force: bool = False, verbose: bool = False) -> str:
    """The test build, libdf11_b200_test.so (test hooks, short wait limit)."""
    if not force and not _stale(TEST_LIB):
        return TEST_LIB
    return _nvcc(TEST_LIB, TEST_FLAGS, verbose)


def build_checked(force: bool = False, verbose: bool = False) -> str:
    """The checked build, libdf11_b200_checked.so (DF11_CHECKED)."""
    if not force and not _stale(CHECKED_LIB):
        return CHECKED_LIB
    return _nvcc(CHECKED_LIB, CHECKED_FLAGS, verbose)


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
    if "--test" in sys.argv:
        print(build_test(force="--force" in sys.argv))
    if "--checked" in sys.argv:
        print(build_checked(force="--force" in sys.argv))
