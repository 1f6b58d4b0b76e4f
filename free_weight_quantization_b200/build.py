"""Builds the CUDA library libhqq_b200.so in-tree with nvcc for sm_100a.

The library is six translation units (the C ABI, the stream engine, the tile engine in two
parts, dequantize + the one-vector forward product, and the tensor-core product of a batch),
compiled in parallel and linked into one shared object.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
UNITS = ["hqq_abi.cu", "hqq_stream.cu", "hqq_tile_a.cu", "hqq_tile_b.cu", "hqq_dequant.cu",
         "hqq_gemm.cu"]
SRCS = [os.path.join(CSRC, u) for u in UNITS]
HDRS = [os.path.join(ROOT, "include", "hqq_b200.h"), os.path.join(CSRC, "hqq_common.cuh"),
        os.path.join(CSRC, "hqq_tile.cuh")]
LIB = os.path.join(HERE, "libhqq_b200.so")
OBJ_DIR = os.path.join(HERE, "_build")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-fmad=false",
              "-prec-div=true", "-prec-sqrt=true", "-ftz=false"]


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _compile(src: str, extra: list[str], verbose: bool) -> str:
    obj = os.path.join(OBJ_DIR, os.path.basename(src) + f".{os.getpid()}.o")
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", os.path.join(ROOT, "include"), "-c", src, "-o", obj]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    return obj


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None) -> str:
    if (not force and os.path.exists(LIB) and not extra
            and os.path.getmtime(LIB) >= max(os.path.getmtime(p) for p in SRCS + HDRS)):
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=len(SRCS)) as ex:
        objs = list(ex.map(lambda s: _compile(s, extra or [], verbose), SRCS))
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, "-shared", *objs, "-o", tmp, "-lcudart"]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    for o in objs:
        os.remove(o)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    import sys
    print(build(force=True, verbose=True, extra=sys.argv[1:]))
