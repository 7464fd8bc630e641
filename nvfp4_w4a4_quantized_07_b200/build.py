"""Build libnvfp4.so (the linear-layer library) and libnvfp4_probes.so (the
peak-measurement kernels bench.py uses) in-tree with nvcc for sm_100a.

Usage: ``python -m nvfp4_w4a4_quantized_07_b200.build [--verbose-ptxas]``.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libnvfp4.so")
SOURCES = [os.path.join(CSRC, "nvfp4_lib.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("ptx.cuh", "quant.cuh", "gemm_common.cuh", "gemm_large.cuh",
                                                 "gemm_decode.cuh", "kv_fp8.cuh")] + [os.path.join(ROOT, "include", "nvfp4.h")]
PROBES_LIB = os.path.join(PKG, "libnvfp4_probes.so")
PROBES_SOURCES = [os.path.join(CSRC, "probes.cu")]
PROBES_DEPS = PROBES_SOURCES + [os.path.join(CSRC, "ptx.cuh")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(verbose_ptxas: bool = False, out: str = LIB, sources=SOURCES) -> list:
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-ftz=false", "-prec-div=true", "-prec-sqrt=true", "-fmad=true",
           "-I" + os.path.join(ROOT, "include"), "-o", out] + list(sources) + \
        ["-lcudart_static", "-ldl", "-lrt", "-lpthread"]
    if verbose_ptxas:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def up_to_date(lib: str = LIB, deps=DEPS) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(d) <= t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if force or verbose_ptxas or not up_to_date():
        subprocess.run(command(verbose_ptxas), check=True)
    return LIB


def build_probes(force: bool = False) -> str:
    if force or not up_to_date(PROBES_LIB, PROBES_DEPS):
        subprocess.run(command(False, PROBES_LIB, PROBES_SOURCES), check=True)
    return PROBES_LIB


if __name__ == "__main__":
    build(force=True, verbose_ptxas="--verbose-ptxas" in sys.argv)
    build_probes(force=True)
    print(LIB)
    print(PROBES_LIB)
