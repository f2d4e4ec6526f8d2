"""Build libdsaidx.so in-tree with nvcc for sm_100a (cross-compiles without a GPU).

Two builds of the same sources: libdsaidx.so, and libdsaidx_checked.so compiled with
-DDSA_DEVICE_CHECKS=1, whose kernels verify the indices they compute on the device (gathered key
rows, candidate positions, bitmap words, output slots) and record a violation in the workspace
status word instead of touching memory outside a buffer.  The checked build is for debugging and
for the test that runs the exact parity cases through it; the package loads it when the
environment variable DSA_LIBRARY is "checked".
"""
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libdsaidx.so")
LIB_CHECKED = os.path.join(HERE, "libdsaidx_checked.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(INCLUDE, "*.h"))) + [os.path.abspath(__file__)]


def up_to_date(lib=LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in deps())


def _command(lib, extra):
    nvcc = os.environ.get("NVCC", "nvcc")
    return [nvcc, *NVCC_FLAGS, *extra, "-I", INCLUDE, "-o", lib + ".tmp", *sources()]


def build(force: bool = False, verbose: bool = False, extra=(), checked: bool = True) -> str:
    """Builds libdsaidx.so (and, with `checked`, libdsaidx_checked.so; the two compile in parallel)."""
    jobs = []
    if force or not up_to_date(LIB):
        jobs.append((LIB, list(extra)))
    if checked and (force or not up_to_date(LIB_CHECKED)):
        jobs.append((LIB_CHECKED, list(extra) + ["-DDSA_DEVICE_CHECKS=1"]))
    procs = []
    for lib, ex in jobs:
        cmd = _command(lib, ex)
        if verbose:
            print(" ".join(cmd))
        procs.append((lib, subprocess.Popen(cmd)))
    for lib, p in procs:
        if p.wait() != 0:
            raise subprocess.CalledProcessError(p.returncode, _command(lib, []))
        os.replace(lib + ".tmp", lib)
    return LIB


if __name__ == "__main__":
    extra = ["-Xptxas", "-v"] if "-v" in sys.argv else []
    print(build(force=True, verbose=True, extra=extra))
