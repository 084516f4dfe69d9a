"""Builds the sm_100a C-ABI library in-tree: vision_language_model_b200/libvlm_b200.so,
and with --debug its checked variant libvlm_b200_debug.so (compiled with
-DVLM_DEBUG: index checks that record a failure code instead of accessing out
of range; see include/vlm_kernels.h).

    python -m vision_language_model_b200.build [--verbose] [--debug]

nvcc cross-compiles for sm_100a without a GPU. Object files go to
vision_language_model_b200/_build/ (git-ignored); the .so sits next to this
file so the binding finds it.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libvlm_b200.so")
DEBUG_LIB = os.path.join(PKG, "libvlm_b200_debug.so")
SOURCES = ["api.cu", "gemm_tcgen05.cu", "attention_tc.cu", "small_kernels.cu", "scatter_noalloc.cu", "frontend.cu",
           "nvfp4.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libvlm_b200.so")


def _stale(out: str, deps) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def build(verbose: bool = False, force: bool = False, ptxas_verbose: bool = False, debug: bool = False) -> str:
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    headers += [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))]
    objdir = os.path.join(PKG, "_build_debug" if debug else "_build")
    lib = DEBUG_LIB if debug else LIB
    os.makedirs(objdir, exist_ok=True)
    flags = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
                    "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]
    if ptxas_verbose:
        flags += ["-Xptxas", "-v"]
    if debug:
        flags += ["-DVLM_DEBUG"]
    objs = []
    for src in SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(objdir, src.replace(".cu", ".o"))
        objs.append(obj)
        if force or _stale(obj, [path] + headers):
            cmd = [nvcc()] + flags + ["-c", path, "-o", obj]
            if verbose:
                print(" ".join(cmd), flush=True)
            subprocess.run(cmd, check=True)
    if force or _stale(lib, objs):
        cmd = [nvcc()] + ARCH + ["-shared", "-o", lib] + objs + ["-lcudart_static", "-ldl", "-lrt", "-lpthread"]
        if verbose:
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)
    return lib


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force="--force" in sys.argv, ptxas_verbose="--ptxas" in sys.argv,
                debug="--debug" in sys.argv))
