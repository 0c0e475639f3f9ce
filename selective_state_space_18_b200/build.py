"""Build ``libssscan.so`` in-tree with nvcc for sm_100a (B200).

    python -m selective_state_space_18_b200.build [--force] [--ptxas-verbose]

The library links the CUDA runtime statically, so it loads without any
LD_LIBRARY_PATH set-up; it shares the primary CUDA context with PyTorch.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libssscan.so")
BOUNDS_LIB = os.path.join(PKG, "libssscan_bounds.so")  # SS_BOUNDS_CHECK debug build

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(INCLUDE, "*.h"))) + [os.path.abspath(__file__)]


def is_stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(d) > t for d in _deps())


def build(force: bool = False, ptxas_verbose: bool = False, verbose: bool = False,
          bounds_check: bool = False) -> str:
    """Compile every CUDA source of the package into ``libssscan.so`` (or, with
    bounds_check, the index-checked debug build ``libssscan_bounds.so``)."""
    lib = BOUNDS_LIB if bounds_check else LIB
    if not force and not is_stale(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [_nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-shared",
           "-Xcompiler", "-fPIC,-fvisibility=hidden", "-cudart", "static",
           "-I", INCLUDE, "-I", CSRC, "--expt-relaxed-constexpr",
           "-o", tmp, *_sources()]
    if bounds_check:
        cmd.insert(1, "-DSS_BOUNDS_CHECK")
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    if verbose:
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    ap.add_argument("--bounds-check", action="store_true", help="the SS_BOUNDS_CHECK debug build")
    args = ap.parse_args()
    print(build(force=args.force, ptxas_verbose=args.ptxas_verbose, verbose=True, bounds_check=args.bounds_check))


if __name__ == "__main__":
    main()
