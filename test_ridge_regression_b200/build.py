"""Builds libgka.so (the C-ABI CUDA library) in-tree with nvcc for sm_100a.

Usage: python -m test_ridge_regression_b200.build [--force]
"""
from __future__ import annotations

import os
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
LIB = PKG / "libgka.so"

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-warn-spills",
]


def _nvcc() -> str:
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    cand = Path(cuda) / "bin" / "nvcc"
    return str(cand) if cand.exists() else "nvcc"


def sources() -> list[Path]:
    return sorted(CSRC.glob("*.cu")) + sorted(CSRC.glob("*.cuh")) + [ROOT / "include" / "gka.h"]


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> Path:
    """Compile csrc/*.cu into libgka.so unless it is newer than every source."""
    if not force and LIB.exists():
        mt = LIB.stat().st_mtime
        if all(p.stat().st_mtime <= mt for p in sources()):
            return LIB
    tmp = LIB.with_suffix(f".so.{os.getpid()}.tmp")
    cmd = [_nvcc(), *NVCC_FLAGS, *(extra or []), "-I", str(ROOT / "include"),
           *[str(p) for p in sorted(CSRC.glob("*.cu"))], "-o", str(tmp)]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else None)
    print(LIB)
