"""Builds libmoe.so in-tree from csrc/ with nvcc for sm_100a.

    python -m mixture_experts_routing_gate_b200.build [--force] [-v]

nvcc cross-compiles without a GPU.  The library links the CUDA runtime statically and reaches the
driver's tensor-map encoder through cudaGetDriverEntryPoint, so it needs no -lcuda at link time.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libmoe.so")
# The test build: the same sources with -DMOE_TEST_HOOKS, which adds moe_test_set_stall (the failure-
# detection hook of tests/test_gpu_failure.py).  The product library has no test hook compiled in.
LIB_TEST_HOOKS = os.path.join(PKG, "libmoe_testhooks.so")
INCLUDE = os.path.join(os.path.dirname(PKG), "include")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC,-O3",
         "-shared", "-I", INCLUDE]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cpp")))


def _deps() -> list[str]:
    return sources() + glob.glob(os.path.join(CSRC, "*.h")) + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(INCLUDE, "*.h"))


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _deps())


def build(force: bool = False, verbose: bool = False, test_hooks: bool = False) -> str:
    """Compiles libmoe.so (or, with test_hooks, libmoe_testhooks.so) unless it is newer than every source."""
    lib = LIB_TEST_HOOKS if test_hooks else LIB
    if not force and up_to_date(lib):
        return lib
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, *FLAGS, *(["-DMOE_TEST_HOOKS"] if test_hooks else []),
           *(["-Xptxas", "-v"] if verbose else []), "-o", tmp, *sources()]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(tmp, lib)
    return lib


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("-v", "--verbose", action="store_true", help="pass -Xptxas -v and print its report")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))


if __name__ == "__main__":
    main()
