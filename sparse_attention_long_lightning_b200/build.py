"""Build libsala.so (all CUDA kernels + the C ABI) for sm_100a, in-tree, and
libsala_debug.so: the same sources with SALA_DEBUG defined, whose kernels check the
indices that data or arithmetic select before each access (a failed check raises
SALA_ERR_BOUNDS instead of faulting).

    python -m sparse_attention_long_lightning_b200.build [--force] [--debug]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libsala.so")
LIB_DEBUG = os.path.join(PKG, "libsala_debug.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _sources():
    out = [os.path.join(ROOT, "include", "sala.h")]
    for f in sorted(os.listdir(CSRC)):
        if f.endswith((".cu", ".cuh")):
            out.append(os.path.join(CSRC, f))
    return out


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile csrc/sala.cu into libsala.so (libsala_debug.so with debug=True, SALA_DEBUG
    defined) unless it is newer than every source."""
    out = LIB_DEBUG if debug else LIB
    if not force and os.path.exists(out):
        t = os.path.getmtime(out)
        if all(os.path.getmtime(s) <= t for s in _sources()):
            return out
    cmd = [nvcc_path(), *ARCH, "-lineinfo", "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
           "-shared", "-I" + os.path.join(ROOT, "include"), os.path.join(CSRC, "sala.cu"),
           "-o", out + ".tmp"]
    if debug:
        cmd.insert(1, "-DSALA_DEBUG")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                debug="--debug" in sys.argv))
