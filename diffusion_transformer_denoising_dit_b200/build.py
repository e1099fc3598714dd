"""Builds libdit.so (the C-ABI library) in-tree for sm_100a with nvcc.

Usage: python -m diffusion_transformer_denoising_dit_b200.build [--force] [--debug]
The library lands next to this file; objects go to <repo>/_build/.  --debug
builds libdit_debug.so instead: the same sources with -DDIT_DEBUG, whose kernels
check their shared-memory, tensor-memory and TMA indices on the device and
record DIT_ERR_BOUNDS in the error word instead of making a bad access (load it
with DIT_LIB_VARIANT=debug).
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
OBJ = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libdit.so")
LIB_DEBUG = os.path.join(PKG, "libdit_debug.so")
SOURCES = ["capi.cu", "rope.cu", "gate.cu", "attn_bf16.cu", "attn_fp8.cu", "fp8_prologue.cu", "selftest.cu",
           "probe.cu"]
HEADERS = ["dit_device.cuh", "dit_internal.h", "attn_kernel.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2,-fvisibility=hidden", "--expt-relaxed-constexpr",
         "-I", os.path.join(ROOT, "include")]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the sm_100a library cannot be built")


def _newest_dep() -> float:
    deps = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "dit.h"), __file__]
    return max(os.path.getmtime(p) for p in deps)


def _compile(src: str, force: bool, debug: bool = False) -> str:
    obj_dir = os.path.join(OBJ, "debug") if debug else OBJ
    out = os.path.join(obj_dir, src.replace(".cu", ".o"))
    path = os.path.join(CSRC, src)
    if not force and os.path.exists(out) and os.path.getmtime(out) >= max(os.path.getmtime(path), _newest_dep()):
        return out
    cmd = [_nvcc(), *ARCH, *FLAGS, *(["-DDIT_DEBUG"] if debug else []), "-c", path, "-o", out]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n{r.stdout}\n{r.stderr}")
    return out


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    os.makedirs(os.path.join(OBJ, "debug") if debug else OBJ, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, force, debug), SOURCES))
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < max(os.path.getmtime(o) for o in objs):
        tmp = lib + ".tmp"
        cmd = [_nvcc(), *ARCH, "-shared", "--cudart", "static", "-o", tmp, *objs]
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, lib)
    if verbose:
        print(lib)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv)
