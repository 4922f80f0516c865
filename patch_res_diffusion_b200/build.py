"""Build the C-ABI library in-tree with nvcc for sm_100a: ``libnpa_b200.so``
and its bounds-checking variant ``libnpa_b200_debug.so`` (the same sources
compiled with NPA_DEBUG_BOUNDS)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OUT = os.path.join(PKG, "libnpa_b200.so")
DEBUG_OUT = os.path.join(PKG, "libnpa_b200_debug.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2", "-shared",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(out: str) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    deps = sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(INCLUDE, "*.h"))
    return any(os.path.getmtime(f) > t for f in deps)


def _compile(out: str, defines, verbose: bool) -> None:
    nvcc = os.environ.get("NVCC", "nvcc")
    cmd = [nvcc, *NVCC_FLAGS, *defines, "-I", INCLUDE, "-o", out + ".tmp", *sources()]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)


def build(force: bool = False, verbose: bool = False) -> str:
    """Builds both libraries if a source is newer (or ``force``); returns the
    path of the normal one."""
    if force or _stale(OUT):
        _compile(OUT, [], verbose)
    if force or _stale(DEBUG_OUT):
        _compile(DEBUG_OUT, ["-DNPA_DEBUG_BOUNDS"], verbose)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
