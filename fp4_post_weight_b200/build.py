"""Build libfocus.so in-tree with nvcc for sm_100a (no PyTorch involved)."""
from __future__ import annotations

import glob
import os
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libfocus.so")
INCLUDE = os.path.join(ROOT, "include")
NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v"]


def sources():
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")) + glob.glob(os.path.join(PKG, "csrc", "*.cuh"))
                  + glob.glob(os.path.join(INCLUDE, "*.h")))


def build(force: bool = False, verbose: bool = False) -> str:
    newest = max(os.path.getmtime(s) for s in sources())
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= newest:
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    cu = sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")))
    tmp = LIB + f".tmp{os.getpid()}"
    # FOCUS_NVTX=0 builds the library without the NVTX ranges around its entry points
    extra = ["-DFOCUS_NO_NVTX"] if os.environ.get("FOCUS_NVTX", "1") == "0" else []
    cmd = [nvcc, *NVCC_FLAGS, *extra, "-I", INCLUDE, *cu, "-o", tmp]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose:
        print(r.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, verbose=True))
