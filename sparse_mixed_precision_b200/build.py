"""Builds libda2.so in-tree with nvcc for sm_100a (B200)."""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libda2.so")
LIB_DEBUG = os.path.join(HERE, "libda2_debug.so")   # DA2_DEBUG: blocking error checks, list checks
SOURCES = ["da2_api.cu", "prep.cu", "draft.cu", "attn_tc.cu", "da2_noalloc.cu", "checks.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(verbose: bool = False, extra: list[str] | None = None, debug: bool = False) -> str:
    """Compile every CUDA source into sparse_mixed_precision_b200/libda2.so (libda2_debug.so
    with DA2_DEBUG defined when debug is set)."""
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    out = LIB_DEBUG if debug else LIB
    cmd = [nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC",
           "-shared", "-I", os.path.join(ROOT, "include"), *(["-DDA2_DEBUG"] if debug else []),
           *(extra or []), *srcs, "-o", out]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(r.stdout + r.stderr, file=sys.stderr)
    return out


if __name__ == "__main__":
    args = [a for a in sys.argv[1:] if a != "--debug"]
    print(build(verbose=True, extra=args, debug="--debug" in sys.argv[1:]))
