"""Build libi8q.so (sm_100a) in-tree with nvcc.

``python -m activation_quantized_gemm_b200.build [--ptxas-verbose]`` compiles
``csrc/i8q.cu`` (one translation unit that includes every kernel) into
``activation_quantized_gemm_b200/libi8q.so``.  The CUDA runtime is linked
statically and the driver is reached through ``cudaGetDriverEntryPoint``, so
the library loads on machines without a GPU driver (its calls then fail with
I8Q_ERR_CUDA).
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC = os.path.join(PKG, "csrc", "i8q.cu")
OUT = os.path.join(PKG, "libi8q.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "--cudart", "static",
    "-I", os.path.join(ROOT, "include"),
]


def sources():
    d = os.path.join(PKG, "csrc")
    return [os.path.join(d, f) for f in sorted(os.listdir(d)) if f.endswith((".cu", ".cuh"))] + [
        os.path.join(ROOT, "include", "i8q.h")]


def up_to_date() -> bool:
    if not os.path.exists(OUT):
        return False
    t = os.path.getmtime(OUT)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(verbose_ptxas: bool = False, force: bool = False) -> str:
    if not force and up_to_date():
        return OUT
    cmd = [NVCC, *FLAGS, SRC, "-o", OUT + ".tmp"]
    if verbose_ptxas:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + r.stdout + r.stderr)
    if verbose_ptxas:
        sys.stderr.write(r.stderr)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(verbose_ptxas="--ptxas-verbose" in sys.argv, force=True))
