"""Build libmla.so in-tree with nvcc for sm_100a (explicit -gencode; no JIT, no torch extension)."""
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
LIB = os.path.join(PKG, "libmla.so")
# the same sources with test hooks compiled in (a switch that stalls a kernel's bounded wait on
# purpose); loaded only by the tests of the wait-expiry path
TEST_LIB = os.path.join(PKG, "libmla_testhooks.so")

NVCC_FLAGS = [
    "-std=c++17", "-O3", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    # only the C ABI is exported: internal symbols (inline statics, kernels' host stubs) stay private
    # to each build, so two builds loaded in one process never share state
    "-Xcompiler", "-fvisibility=hidden",
]


def _nvcc():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise FileNotFoundError("nvcc not found: the CUDA toolkit is needed to build libmla.so")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh")) +
                  glob.glob(os.path.join(INCLUDE, "*.h")))


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in sources())


def build_test_hooks(force: bool = False, verbose: bool = False) -> str:
    """Compile the test-hooks variant of the library (-DMLA_TEST_HOOKS) into libmla_testhooks.so."""
    return build(force, verbose, ["-DMLA_TEST_HOOKS"], TEST_LIB)


def build(force: bool = False, verbose: bool = False, extra_flags=None, lib: str = LIB) -> str:
    """Compile csrc/mla_api.cu (which includes every kernel) into `lib` (libmla.so); return its path."""
    if not force and up_to_date(lib):
        return lib
    cmd = [_nvcc(), *NVCC_FLAGS, *(extra_flags or []), "-I", INCLUDE, "-I", CSRC,
           "-o", lib + ".tmp", os.path.join(CSRC, "mla_api.cu")]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose and (res.stdout or res.stderr):
        print(res.stdout, res.stderr, file=sys.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
