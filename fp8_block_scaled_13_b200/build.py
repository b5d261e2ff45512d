"""Build the CUDA library libpuro_fp8.so in-tree (nvcc, sm_100a only)."""
from __future__ import annotations

import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB_PATH = os.path.join(HERE, "libpuro_fp8.so")
SOURCES = ["puro_fp8.cu"]
DEPS = ["puro_fp8.cu", "common.cuh", "quant.cuh", "gemm.cuh"]
HEADER = os.path.join(ROOT, "include", "puro_fp8.h")


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA library cannot be built")


def nvcc_command(out: str, verbose_ptxas: bool = False) -> list:
    cmd = [
        nvcc_path(),
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC,-fvisibility=hidden",
        "-shared", "-Xlinker", "--exclude-libs,ALL",
        "-o", out,
    ]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    return cmd


def stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    deps = [os.path.join(CSRC, d) for d in DEPS] + [HEADER]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    if force or stale():
        tmp = LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.run(nvcc_command(tmp, verbose_ptxas), check=True)
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas=True))
