"""Build libgdn_b200.so from csrc/ with nvcc for sm_100a (in-tree).

    python -m gated_delta_rule_fg_b200.build [--verbose-ptxas]
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SO = os.path.join(HERE, "libgdn_b200.so")
SO_BOUNDS = os.path.join(HERE, "libgdn_b200_bounds.so")     # -DGDN_DEBUG_BOUNDS
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def headers():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cuh")) + glob.glob(os.path.join(HERE, "csrc", "*.h")) +
                  glob.glob(os.path.join(ROOT, "include", "*.h")))


def up_to_date(so: str = SO) -> bool:
    if not os.path.exists(so):
        return False
    t = os.path.getmtime(so)
    return all(os.path.getmtime(f) <= t for f in sources() + headers())


def build(force: bool = False, ptxas_verbose: bool = False, debug_bounds: bool = False) -> str:
    """The library (or, with debug_bounds, its bounds-checking build: -DGDN_DEBUG_BOUNDS, the
    same ABI in libgdn_b200_bounds.so)."""
    so = SO_BOUNDS if debug_bounds else SO
    if not force and up_to_date(so):
        return so
    tmp = so + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
           "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"),
           "-o", tmp, *sources(), "-lcudart"]
    if debug_bounds:
        cmd.insert(1, "-DGDN_DEBUG_BOUNDS")
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(tmp, so)
    return so


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv, debug_bounds="--debug-bounds" in sys.argv))
