"""Build libw8a8.so in-tree with nvcc for sm_100a (no JIT cache, no torch build
machinery).  ``python -m w8a8_quantized_linear_b200._build`` or
``__graft_entry__.build()``."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libw8a8.so")
# the same sources with the device-side index checks (W8A8_DEBUG_CHECKS=1)
LIB_DEBUG = os.path.join(PKG, "libw8a8_debug.so")
MAIN = os.path.join(CSRC, "w8a8.cu")
HEADERS = [os.path.join(ROOT, "include", "w8a8.h")] + [
    os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cuh", ".cu"))]

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(out: str = LIB, extra=()) -> list:
    return [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
            "-I", os.path.join(ROOT, "include"), "-o", out, MAIN, *extra]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(h) <= t for h in HEADERS)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Build libw8a8.so, or with debug=True libw8a8_debug.so (device-side
    index checks that record an error code instead of faulting)."""
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(lib):
        return lib
    tmp = lib + ".tmp.%d" % os.getpid()
    extra = (["-Xptxas", "-v"] if verbose else []) + (["-DW8A8_DEBUG_CHECKS=1"] if debug else [])
    cmd = command(tmp, extra)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building %s" % os.path.basename(lib))
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
