"""Builds libcoda.so (the C-ABI CUDA library) in-tree for sm_100a.

    python -m gemm_epilogue_transformer_02_b200.build [--verbose]

The library is one translation unit (csrc/coda.cu) compiled with nvcc for
compute_100a / sm_100a, with the CUDA runtime linked statically so the shared
object only needs the NVIDIA driver at run time.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libcoda.so")

SOURCES = ["coda.cu"]
DEPS = ["coda.cu", "coda_device.cuh", "coda_gemm.cuh", "coda_rowops.cuh", "coda_block.cuh", "coda_grouped.cuh"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found (set NVCC or install the CUDA toolkit)")


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    srcs = [os.path.join(CSRC, d) for d in DEPS] + [os.path.join(INCLUDE, "coda.h")]
    return all(os.path.getmtime(s) <= t for s in srcs)


def build(verbose: bool = False, force: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [
        nvcc_path(),
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-std=c++17", "-lineinfo",
        "-Xcompiler", "-fPIC", "-shared",
        "-cudart", "static",
        "--expt-relaxed-constexpr",
        "-I", INCLUDE,
        "-o", LIB + ".tmp",
    ]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    proc = subprocess.run(cmd, capture_output=True, text=True)
    if proc.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + proc.stdout + proc.stderr)
    if verbose:
        sys.stderr.write(proc.stdout + proc.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force=True)
    print(LIB)
