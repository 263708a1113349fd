"""Build libmoedc.so (the C-ABI CUDA library) in-tree with nvcc for sm_100a.

    python -m combine_topk_ids_scan_b200.build [--verbose] [--force] [--debug | --trace]

No fast-math: the FP8 / NVFP4 scales use IEEE round-to-nearest division and
the combine relies on exact fused multiply-adds.
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(PKG, "libmoedc.so")
# the same sources with device index checks (-DMOE_DEBUG_CHECKS)
DEBUG_LIB_PATH = os.path.join(PKG, "libmoedc_debug.so")
# the same sources with per-CTA trace records (-DMOE_TRACE)
TRACE_LIB_PATH = os.path.join(PKG, "libmoedc_trace.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
              "--expt-relaxed-constexpr", "-Xcompiler", "-fvisibility=hidden"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs() -> list[str]:
    return (sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")))
            + sorted(glob.glob(os.path.join(CSRC, "*.h")))
            + sorted(glob.glob(os.path.join(INCLUDE, "*.h"))) + [os.path.abspath(__file__)])


def up_to_date(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, debug: bool = False,
          trace: bool = False) -> str:
    """Build libmoedc.so; with debug=True libmoedc_debug.so (device index
    checks, see moe_debug_violations in moe_dc.h); with trace=True
    libmoedc_trace.so (per-CTA trace records, see moe_trace_attach)."""
    if debug and trace:
        raise ValueError("one build option at a time")
    path = DEBUG_LIB_PATH if debug else TRACE_LIB_PATH if trace else LIB_PATH
    if not force and up_to_date(path):
        return path
    tmp = path + f".tmp{os.getpid()}"
    defines = ["-DMOE_DEBUG_CHECKS"] if debug else ["-DMOE_TRACE"] if trace else []
    cmd = [_nvcc(), *ARCH_FLAGS, *NVCC_FLAGS, *defines,
           "-I", INCLUDE, "-I", CSRC, "-o", tmp, *sources()]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, path)
    return path


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--debug", action="store_true",
                    help="build libmoedc_debug.so with device index checks")
    ap.add_argument("--trace", action="store_true",
                    help="build libmoedc_trace.so with per-CTA trace records")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, debug=a.debug, trace=a.trace))
    sys.exit(0)
