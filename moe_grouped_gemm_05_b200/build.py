"""Builds libdg.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: ``python -m moe_grouped_gemm_05_b200.build [--verbose]``.  The library
is written next to this file so that it travels with the source tree.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libdg.so")
SOURCES = ["dg_api.cu"]
DEPS = ["dg_api.cu", "fp8_gemm_kernel.cuh", "ptx.cuh", "quant_kernel.cuh", "moe_kernels.cuh"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def flags(ptxas_verbose: bool = False) -> list[str]:
    f = [
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-lineinfo", "-std=c++17",
        "-Xcompiler", "-fPIC", "-shared",
        "-I", os.path.join(ROOT, "include"),
        "--expt-relaxed-constexpr",
    ]
    if ptxas_verbose:
        f += ["-Xptxas", "-v"]
    return f


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    paths = [os.path.join(CSRC, s) for s in DEPS] + [os.path.join(ROOT, "include", "dg.h")]
    return all(os.path.getmtime(p) <= t for p in paths)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    cmd = [nvcc_path(), *flags(verbose), "-o", LIB + ".tmp", *[os.path.join(CSRC, s) for s in SOURCES]]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}): {' '.join(cmd)}")
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
