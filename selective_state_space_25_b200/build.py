"""Builds libssmscan.so (the CUDA kernels + C ABI) in-tree with nvcc for
sm_100a.  Run directly (``python -m selective_state_space_25_b200.build``) or
through ``__graft_entry__.build()``.  No GPU is needed to build."""
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
LIB = os.path.join(PKG, "libssmscan.so")
# the debug-bounds build: every kernel checks its global indices (SSM_DEBUG_BOUNDS)
LIB_DEBUG = os.path.join(PKG, "libssmscan_debug.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
         "--expt-relaxed-constexpr", "-Xcompiler", "-Wall"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(INCLUDE, "*.h")))


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in deps())


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False,
          debug_bounds: bool = False) -> str:
    """Builds libssmscan.so, or with debug_bounds libssmscan_debug.so (the
    same sources compiled with SSM_DEBUG_BOUNDS)."""
    lib = LIB_DEBUG if debug_bounds else LIB
    if not force and up_to_date(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    defs = ["-DSSM_DEBUG_BOUNDS"] if debug_bounds else []
    cmd = [nvcc(), *ARCH, *FLAGS, *defs, f"-I{INCLUDE}", f"-I{CSRC}", *sources(), "-o", tmp]
    if ptxas_info:
        cmd.insert(1, "-Xptxas=-v")
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed ({r.returncode}):\n{r.stdout}\n{r.stderr}")
    if verbose or ptxas_info:
        sys.stdout.write(r.stdout + r.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    for dbg in (False, True):
        print("built", build(force="--force" in sys.argv, verbose=True,
                             ptxas_info="--ptxas-info" in sys.argv, debug_bounds=dbg))
