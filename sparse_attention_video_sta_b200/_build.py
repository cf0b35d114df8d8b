"""Build libsta.so (the C-ABI STA library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(PKG_DIR, "libsta.so")
# The same library with the device-side checks of every plan index compiled in
# (STA_DEBUG_BOUNDS; see csrc/sta_bounds.cuh).
DEBUG_LIB_PATH = os.path.join(PKG_DIR, "libsta_debug.so")

SOURCES = ["sta_api.cu", "sta_permute.cu", "sta_forward.cu", "sta_backward.cu", "sta_search.cu", "sta_pipe.cu", "sta_noalloc.cu"]
HEADERS = ["sta_internal.h", "sta_ptx.cuh", "sta_raster.cuh", "sta_wait.cuh", "sta_bounds.cuh"]

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared",
]


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(INCLUDE, "sta.h"))
    return files


def up_to_date(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return False
    t = os.path.getmtime(path)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def _compile(path: str, extra, verbose: bool):
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = path + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, *extra, "-I", INCLUDE, "-I", CSRC,
           *[os.path.join(CSRC, f) for f in SOURCES], "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, path)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Build libsta.so (and, with debug=True, also libsta_debug.so)."""
    if force or not up_to_date(LIB_PATH):
        _compile(LIB_PATH, [], verbose)
    if debug and (force or not up_to_date(DEBUG_LIB_PATH)):
        _compile(DEBUG_LIB_PATH, ["-DSTA_DEBUG_BOUNDS"], verbose)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
