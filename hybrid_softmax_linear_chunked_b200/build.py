"""Build step: compile librehyat.so for sm_100a in-tree (hybrid_softmax_linear_chunked_b200/_lib)."""
from __future__ import annotations

import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "rehyat.cu")
OUT = os.path.join(HERE, "_lib", "librehyat.so")
# The debug-bounds variant: every TMA coordinate and global store index of the forward kernels
# checked, failures reported through rehyat_sync_status (REHYAT_ERR_BOUNDS) instead of faulting.
OUT_DEBUG = os.path.join(HERE, "_lib", "librehyat_debug.so")

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
              "-shared", "-Xcompiler", "-fPIC"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources() -> list[str]:
    d = os.path.join(HERE, "csrc")
    inc = os.path.join(os.path.dirname(HERE), "include", "rehyat.h")
    return [os.path.join(d, f) for f in os.listdir(d)] + [inc]


def build(force: bool = False, verbose: bool = False, debug_bounds: bool = False) -> str:
    """Compile the library (or, with debug_bounds, its bounds-checking variant) if any source is
    newer than the built .so; return its path."""
    out = OUT_DEBUG if debug_bounds else OUT
    if not force and os.path.exists(out):
        built = os.path.getmtime(out)
        if all(os.path.getmtime(s) <= built for s in _sources()):
            return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + ".tmp"
    flags = NVCC_FLAGS + (["-DREHYAT_DEBUG_BOUNDS"] if debug_bounds else [])
    cmd = [_nvcc(), *flags, "-o", tmp, SRC]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed:\n{res.stdout}\n{res.stderr}")
    os.replace(tmp, out)
    if verbose:
        print(res.stderr)
    return out


if __name__ == "__main__":
    print(build(force=True, verbose=True))
    print(build(force=True, debug_bounds=True))
