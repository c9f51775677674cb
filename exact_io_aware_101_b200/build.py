"""Build libexattn.so in-tree with nvcc for sm_100a.

Usage: ``python -m exact_io_aware_101_b200.build [--force] [--verbose]``.
The library links the CUDA runtime statically and reaches the driver's tensor
map encoder through cudaGetDriverEntryPoint, so it needs only the NVIDIA
driver at run time.  Each kernel file compiles to its own object (in parallel,
in a temporary directory), then one link makes the library.

``build_test_lib()`` makes a second library, used only by tests: the same
sources with every wait limited to TEST_WAIT_CYCLES instead of about 1.5 s,
with the producers of the prefill and decode kernels stopping before ring index
TEST_WITHHOLD (so that the kernels' waits run out on purpose and their abort
paths run).  The product library is never built with these switches.
"""
from __future__ import annotations

import concurrent.futures as cf
import glob
import os
import subprocess
import sys
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libexattn.so")
TEST_LIB = os.path.join(HERE, "libexattn_testbuild.so")
INCLUDE = os.path.join(ROOT, "include")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]
# The test build: ~1 ms waits, producers stop before ring index 2 (the
# prefill's second K tile; the decode's third page of a chunk).
TEST_WAIT_CYCLES = 2000000
TEST_WITHHOLD = 2
TEST_FLAGS = ["-DEXATTN_WAIT_LIMIT_CYCLES=%dLL" % TEST_WAIT_CYCLES,
              "-DEXATTN_TEST_WITHHOLD=%d" % TEST_WITHHOLD]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (_sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + glob.glob(os.path.join(INCLUDE, "*.h")))


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _up_to_date(target: str) -> bool:
    if not os.path.exists(target):
        return False
    t = os.path.getmtime(target)
    return all(os.path.getmtime(p) <= t for p in _deps())


def _link(target: str, flags, verbose: bool) -> str:
    with tempfile.TemporaryDirectory(prefix="exattn_build_") as objdir:
        return _compile_and_link(target, flags, objdir, verbose)


def _compile_and_link(target: str, flags, objdir: str, verbose: bool) -> str:
    base = [nvcc()] + NVCC_FLAGS + list(flags)
    if verbose:
        base.insert(1, "-Xptxas=-v")

    def compile_one(src):
        obj = os.path.join(objdir, os.path.basename(src)[:-3] + ".o")
        cmd = base + ["-c", src, "-o", obj]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.check_call(cmd)
        return obj

    workers = max(1, min(len(_sources()), os.cpu_count() or 1))
    with cf.ThreadPoolExecutor(workers) as ex:
        objs = list(ex.map(compile_one, _sources()))
    tmp = target + ".tmp%d" % os.getpid()
    subprocess.check_call([nvcc()] + NVCC_FLAGS[:2] + ["-shared", "-o", tmp] + objs)
    os.replace(tmp, target)
    return target


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    """Compile every kernel file and the C ABI into libexattn.so; returns its path."""
    if not force and not extra and _up_to_date(LIB):
        return LIB
    return _link(LIB, extra, verbose)


def build_test_lib(force: bool = False, verbose: bool = False) -> str:
    """The test build of the library (see the module docstring); returns its path."""
    if not force and _up_to_date(TEST_LIB):
        return TEST_LIB
    return _link(TEST_LIB, TEST_FLAGS, verbose)


if __name__ == "__main__":
    force, verbose = "--force" in sys.argv, "--verbose" in sys.argv
    print(build(force=force, verbose=verbose))
    print(build_test_lib(force=force, verbose=verbose))
