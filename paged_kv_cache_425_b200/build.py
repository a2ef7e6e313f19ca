"""Build libpa.so in-tree with nvcc for sm_100a.

    python paged_kv_cache_425_b200/build.py [--force] [--ptxas-verbose]

(Run it by path: importing the package itself loads the library this script
builds.)

The library holds the CUDA kernels, the C ABI of include/pa_api.h and the
host block allocator of include/pa_alloc.h.  It links the CUDA runtime
statically and reaches the driver's tensor-map encoder at run time, so it
loads (and the allocator runs) on a machine without a GPU.
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libpa.so")
SOURCES = [os.path.join(CSRC, f) for f in ("pa_api.cu", "pa_alloc.cc", "pa_sim.cc")]
# every file the library is built from: a change to any header rebuilds it
DEPS = sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)) + sorted(
    os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE))

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in DEPS if os.path.exists(p))


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    if not (force or stale()):
        return LIB
    tmp = LIB + f".{os.getpid()}.tmp"
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-o", tmp, *SOURCES]
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    args = ap.parse_args(argv)
    print(build(args.force, args.ptxas_verbose))


if __name__ == "__main__":
    sys.exit(main())
