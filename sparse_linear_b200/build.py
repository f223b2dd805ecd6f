"""Builds libactsparse.so in-tree with nvcc for sm_100a (B200)."""
from __future__ import annotations

import glob
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libactsparse.so")
# the same library with index checks (-DAS_BOUNDS_CHECK): a failed check
# skips the access and records AS_ERR_BOUNDS (for tests, not for production)
LIB_CHECKED = os.path.join(HERE, "libactsparse_checked.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
    "-Xptxas", "-warn-spills",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")) + glob.glob(os.path.join(CSRC, "*.cuh"))
                  + [os.path.join(HERE, "..", "include", "actsparse.h")])


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(s) > t for s in sources())


def _compile(lib: str, extra: list[str], verbose: bool) -> None:
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, *extra, *(["-Xptxas", "-v"] if verbose else []),
           os.path.join(CSRC, "actsparse.cu"), "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if a source is newer than it (or ``force``)."""
    if force or stale(LIB):
        _compile(LIB, [], verbose)
    return LIB


def build_checked(force: bool = False) -> str:
    """Compile the index-checked library (-DAS_BOUNDS_CHECK) if stale."""
    if force or stale(LIB_CHECKED):
        _compile(LIB_CHECKED, ["-DAS_BOUNDS_CHECK"], False)
    return LIB_CHECKED


if __name__ == "__main__":
    import sys
    build(force=True, verbose="-v" in sys.argv)
    print(LIB)
    if "--checked" in sys.argv:
        print(build_checked(force=True))
