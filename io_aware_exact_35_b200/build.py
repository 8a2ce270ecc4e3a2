"""Build libfa_b200.so in-tree with nvcc for sm_100a.

    python -m io_aware_exact_35_b200.build [--verbose] [--debug]

The library is one CUDA translation unit (csrc/fa_lib.cu) linked against the
static CUDA runtime; it needs no PyTorch headers.  The output lands in
io_aware_exact_35_b200/lib/ so that it travels with the source tree.

``--debug`` builds lib/libfa_b200_debug.so with -DFA_DEBUG: the kernels check
every computed global address and TMA coordinate and record FA_ERR_BOUNDS in
the device error word instead of making a bad access (see sm100.cuh).  Point
FA_B200_LIBRARY at it to run a program against the checked kernels.
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIBDIR = os.path.join(PKG, "lib")
LIB = os.path.join(LIBDIR, "libfa_b200.so")
DEBUG_LIB = os.path.join(LIBDIR, "libfa_b200_debug.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cuh", ".h"))) + [os.path.join(ROOT, "include", "fa_b200.h")]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(verbose: bool = False, force: bool = False, debug: bool = False) -> str:
    lib = DEBUG_LIB if debug else LIB
    if not force and up_to_date(lib):
        return lib
    os.makedirs(LIBDIR, exist_ok=True)
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH_FLAGS, "-O3", "-std=c++17", "-lineinfo", "--use_fast_math",
           "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
           *(["-DFA_DEBUG"] if debug else []),
           os.path.join(CSRC, "fa_lib.cu"), "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError(f"nvcc failed to build {os.path.basename(lib)}")
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--debug", action="store_true")
    a = ap.parse_args()
    print(build(verbose=a.verbose, force=a.force, debug=a.debug))
