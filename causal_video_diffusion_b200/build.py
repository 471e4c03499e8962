"""Build ``libunstep.so`` (the sm_100a CUDA library behind include/unstep.h) in-tree.

``python -m causal_video_diffusion_b200.build [--force]``.  nvcc cross-compiles for sm_100a
without a GPU; the shared library links the CUDA runtime statically and needs no libcuda at link
time (the TMA descriptor encoder is fetched from the driver at run time).
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libunstep.so")
# the same library with the kernels' index checks compiled in (-DUNSTEP_DEBUG): a failed check
# records UNSTEP_ERR_DEVICE_BOUNDS in the cache's error word instead of touching memory
DEBUG_LIB = os.path.join(PKG, "libunstep_debug.so")
SOURCES = ["api.cu", "rope_append.cu", "window_attn.cu", "lowrank_gemm.cu", "renoise.cu",
           "conv3d.cu", "gemm2sm.cu"]
HEADERS = ["internal.h", "limits.h", "gemm.h", "conv3d.h", "sm100.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
         "--expt-relaxed-constexpr", "-Xptxas", "-v", "-I", os.path.join(ROOT, "include")]


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "unstep.h"))
    return files


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = DEBUG_LIB if debug else LIB
    if not (force or needs_build(lib)):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    extra = ["-DUNSTEP_DEBUG"] if debug else []
    cmd = [NVCC, *ARCH, *FLAGS, *extra, "-o", tmp, *[os.path.join(CSRC, s) for s in SOURCES]]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError(f"nvcc failed building {os.path.basename(lib)}")
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
