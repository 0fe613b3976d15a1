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
# the same library with device-side bounds checks (E2D2_DEBUG): selected by E2D2_DEBUG=1
DEBUG_LIBRARY = PKG / "libe2d2_attn_debug.so"
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


def up_to_date(lib: Path = LIBRARY) -> bool:
    if not lib.exists():
        return False
    t = lib.stat().st_mtime
    return all(p.stat().st_mtime <= t for p in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False, extra=(), debug: bool = False) -> Path:
    """Builds the library (debug=True: the E2D2_DEBUG variant with device bounds checks)."""
    lib = DEBUG_LIBRARY if debug else LIBRARY
    if not force and up_to_date(lib):
        return lib
    flags = ["-DE2D2_DEBUG"] if debug else []
    cmd = [nvcc(), *NVCC_FLAGS, *flags, *extra, "-I", str(ROOT / "include"), "-I", str(CSRC),
           *map(str, SOURCES), "-o", str(lib)]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    return lib


def build_all(force: bool = False, verbose: bool = False) -> None:
    build(force=force, verbose=verbose)
    build(force=force, verbose=verbose, debug=True)


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [], debug="--debug" in sys.argv)
