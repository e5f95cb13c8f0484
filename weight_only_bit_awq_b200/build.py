"""Build libawq_b200.so in-tree with nvcc for sm_100a.

Usage: python weight_only_bit_awq_b200/build.py [--force] [--verbose]
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libawq_b200.so")
# The debug build (-DAWQ_DEBUG): every guarded global and shared access of the
# pack, dequant, GEMV and GEMM kernels checks its index range first and records
# AWQ_ERR_BOUNDS instead of faulting. Same entry points, separate file.
LIB_DEBUG = os.path.join(PKG, "libawq_b200_debug.so")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ARCH + ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC]
# The pack kernel must not contract fp64 operations (bit-exact quantization).
PER_FILE = {"pack.cu": ["--fmad=false"]}
SOURCES = ["abi.cu", "pack.cu", "gemv.cu", "gemm_tc.cu", "gemm_fp8.cu", "no_alloc.cu"]
HEADERS = ["awq_internal.cuh", "sm100_ptx.cuh", "gemv_common.cuh"]


def _newest_input() -> float:
    paths = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "awq.h"), __file__]
    return max(os.path.getmtime(p) for p in paths)


def _compile(src: str, verbose: bool, debug: bool = False) -> str:
    obj = os.path.join(BUILD, ("debug_" if debug else "") + src.replace(".cu", ".o"))
    cmd = [NVCC, *COMMON, *PER_FILE.get(src, []), *(["-DAWQ_DEBUG"] if debug else []), "-c", os.path.join(CSRC, src),
           "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose:
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= _newest_input():
        return lib
    os.makedirs(BUILD, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, debug), SOURCES))
    tmp = lib + f".tmp{os.getpid()}"
    r = subprocess.run([NVCC, *ARCH, "-shared", "-o", tmp, *objs], capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))
