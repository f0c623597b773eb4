"""Build ``libgdn.so`` in-tree with nvcc for sm_100a.

    python -m linear_attention_recurrence_04_b200.build [--force] [-DNAME=VALUE ...]

The library is written next to this file. Extra ``-D`` definitions select
kernel tuning constants (rows per warp task, CTA size); the defaults are the
measured best.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys
from typing import List, Optional

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(PKG, "libgdn.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def sources() -> List[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs() -> List[str]:
    return (sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + glob.glob(os.path.join(INCLUDE, "*.h")))


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def build(output: str = LIBRARY, defines: Optional[List[str]] = None, force: bool = False,
          verbose: bool = False) -> str:
    """Compile every ``csrc/*.cu`` into one shared library; return its path."""
    defines = defines or []
    if (not force and not defines and os.path.exists(output)
            and os.path.getmtime(output) >= max(os.path.getmtime(p) for p in _inputs())):
        return output
    cmd = [nvcc(), *NVCC_FLAGS, "-I", INCLUDE, "-I", CSRC, *defines]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += ["-o", output, *sources()]
    subprocess.run(cmd, check=True)
    return output


if __name__ == "__main__":
    args = sys.argv[1:]
    defs = [a for a in args if a.startswith("-D")]
    out = LIBRARY
    for a in args:
        if a.startswith("--out="):
            out = a.split("=", 1)[1]
    print(build(out, defs, force="--force" in args, verbose="--verbose" in args))
