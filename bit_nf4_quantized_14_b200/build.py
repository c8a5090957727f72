"""Build the library in place: libqlora_nf4.so next to this file, for sm_100a only.

    python -m bit_nf4_quantized_14_b200.build [--force]

nvcc cross-compiles without a GPU. The CUDA runtime is linked statically; the driver's tensor-map
encoder is looked up at run time, so the library loads (and its host-only calls work) on machines
without a GPU.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libqlora_nf4.so")
SOURCES = [os.path.join(HERE, "csrc", f) for f in ("api.cu", "codebook.cpp")]
HEADERS = [os.path.join(HERE, "csrc", f) for f in ("common.cuh", "codec.cuh", "codebook_study.cuh", "gemm_sm100.cuh", "gemm_nf4w.cuh",
                                                              "gemv_nf4.cuh", "adamw.cuh", "selftest.cuh", "decode_nf4.cuh")] + [
    os.path.join(ROOT, "include", "qlora_nf4.h")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
         "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v", "-I", os.path.join(ROOT, "include")]


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in SOURCES + HEADERS)


def build(force: bool = False, verbose: bool = False) -> str:
    if force or stale():
        cmd = [NVCC] + FLAGS + SOURCES + ["-o", LIB]
        res = subprocess.run(cmd, capture_output=True, text=True)
        if res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
            raise RuntimeError("nvcc failed building libqlora_nf4.so")
        if verbose:
            sys.stderr.write(res.stderr)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
