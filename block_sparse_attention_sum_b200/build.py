"""Build the sm_100a CUDA library (libsolattn.so) in-tree with nvcc.

Usage: python -m block_sparse_attention_sum_b200.build [--verbose]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libsolattn.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)
# the same library with the device-side bounds checks compiled in (-DSOL_ATTN_DEBUG_BOUNDS)
DEBUG_LIB_PATH = os.path.join(HERE, "libsolattn_debug.so")
SOURCES = ["api.cu", "summary.cu", "route_tc.cu", "attn_fwd.cu", "splitkv.cu", "sol2_tail.cu", "sol2_tail_tc.cu", "noalloc.cu",
           "quant_fp8.cu", "attn_fwd_fp8.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found")
    return path


def build(verbose: bool = False, force: bool = False, debug_bounds: bool = False) -> str:
    """Compile the library (or its bounds-checked debug variant) unless it is newer than its sources."""
    out = DEBUG_LIB_PATH if debug_bounds else LIB_PATH
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    deps = srcs + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")]
    deps.append(os.path.join(INCLUDE, "sol_attn.h"))
    if not force and os.path.exists(out):
        t = os.path.getmtime(out)
        if all(os.path.getmtime(d) <= t for d in deps):
            return out
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC,-O3",
           "--expt-relaxed-constexpr", f"-I{INCLUDE}", f"-I{CSRC}", "-o", out + ".tmp", *srcs]
    if debug_bounds:
        cmd.insert(1, "-DSOL_ATTN_DEBUG_BOUNDS")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force=True, debug_bounds="--debug-bounds" in sys.argv))
