"""Build the C-ABI shared library ``libdsa_b200.so`` for sm_100a (in-tree).

    python -m long_context_decode_indexer_b200.build [--force] [--ptxas-verbose]

nvcc cross-compiles without a GPU.  The library links the CUDA runtime
statically and reaches the driver only through cudaGetDriverEntryPoint, so
it loads on a machine without a GPU (every compute call then fails with
DSA_ERR_CUDA).
"""
from __future__ import annotations

import argparse
import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libdsa_b200.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) \
        + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False, out: str = None, defines=()) -> str:
    """Compile the library (to `out`, default the in-tree libdsa_b200.so),
    with extra -D `defines`."""
    target = out or LIB
    if not force and out is None and not defines and not _stale():
        return LIB
    tmp = target + ".tmp%d" % os.getpid()
    cmd = [NVCC, *ARCH_FLAGS, "-lineinfo", "-O3", "-std=c++17", "--expt-relaxed-constexpr",
           "-Xcompiler", "-fPIC", "-shared", "-I", INCLUDE, "-I", CSRC,
           *["-D" + d for d in defines], "-o", tmp, *sources()]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force or args.ptxas_verbose, verbose_ptxas=args.ptxas_verbose))
    sys.exit(0)
