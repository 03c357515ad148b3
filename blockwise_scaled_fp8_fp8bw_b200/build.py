"""Builds libfp8bw.so (the C-ABI library) in-tree for sm_100a with nvcc.

Usage: python -m blockwise_scaled_fp8_fp8bw_b200.build [--force]
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(ROOT, "_build")
LIB = os.path.join(HERE, "libfp8bw.so")
SOURCES = ["quant.cu", "quant_tensor.cu", "gemm.cu", "attention.cu", "decode.cu", "api.cu"]
HEADERS = ["common.cuh", "tmap.cuh", "blockquant.cuh"]

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
# IEEE division and denormals stay on (no --use_fast_math, no -ftz): the
# quantizers must be bit-exact.
FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo",
         "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "-ftz=false", "-prec-div=true", "-prec-sqrt=true"]


def _deps():
    return [os.path.join(CSRC, h) for h in HEADERS] + [
        os.path.join(ROOT, "include", "fp8bw.h"), os.path.abspath(__file__)]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _compile(src, force):
    obj = os.path.join(OBJ, os.path.splitext(src)[0] + ".o")
    deps = [os.path.join(CSRC, src)] + _deps()
    if force or _stale(obj, deps):
        cmd = [NVCC, *FLAGS, "-c", os.path.join(CSRC, src), "-o", obj]
        subprocess.check_call(cmd)
    return obj


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(OBJ, exist_ok=True)
    with ThreadPoolExecutor(max_workers=len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, force), SOURCES))
    if force or _stale(LIB, objs):
        tmp = LIB + ".tmp"
        subprocess.check_call([NVCC, "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
                               "-Xlinker", "--exclude-libs,ALL", "-Xlinker", "-Bsymbolic",
                               "-o", tmp, *objs])
        os.replace(tmp, LIB)
    if verbose:
        print(LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
