"""Builds the in-tree CUDA library ``libe2d2_attn.so`` for B200 (sm_100a) with nvcc."""
from __future__ import annotations

import os
import subprocess
import sys
from pathlib import Path

PKG = Path(__file__).resolve().parent
ROOT = PKG.parent
CSRC = PKG / "csrc"
LIBRARY = PKG / "libe2d2_attn.so"
SOURCES = [CSRC / "e2d2_api.cu"]
HEADERS = sorted(CSRC.glob("*.cuh")) + [ROOT / "include" / "e2d2_attn.h"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    cand = Path(os.environ.get("CUDA_HOME", "/usr/local/cuda")) / "bin" / "nvcc"
    return str(cand) if cand.exists() else "nvcc"


def up_to_date() -> bool:
    if not LIBRARY.exists():
        return False
    t = LIBRARY.stat().st_mtime
    return all(p.stat().st_mtime <= t for p in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False, extra=()) -> Path:
    if not force and up_to_date():
        return LIBRARY
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", str(ROOT / "include"), "-I", str(CSRC),
           *map(str, SOURCES), "-o", str(LIBRARY)]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    return LIBRARY


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
