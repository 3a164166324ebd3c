"""Build the CUDA library ``libaxis_attn.so`` in-tree with nvcc for sm_100a.

Usage: ``python -m causal_attention_fwd_b200.build [--force] [--verbose]``.
nvcc cross-compiles without a GPU.  The library links the CUDA runtime
statically and reaches the driver's tensor-map encoder through
cudaGetDriverEntryPoint, so it needs no libcuda at link time.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libaxis_attn.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(ROOT, "include", "axis_attn.h")])


def build(force: bool = False, verbose: bool = False, extra=(), out: str | None = None) -> str:
    """Compile ``csrc/axis_attn.cu`` into ``out`` (default: the in-tree
    ``libaxis_attn.so``).  ``extra`` adds nvcc flags (e.g. ``-D`` switches
    for a test-only build, which then goes to its own ``out``)."""
    lib = out or LIB
    newest = max(os.path.getmtime(p) for p in sources())
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= newest and not extra:
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, *(["-Xptxas", "-v"] if verbose else []), *extra,
           "-o", tmp, os.path.join(CSRC, "axis_attn.cu")]
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv))
