"""Build the sm_100a shared library ``libmoe_grouped.so`` in-tree with nvcc.

Usage: ``python -m mixture_experts_grouped_top_b200.build [--force] [--verbose]``.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libmoe_grouped.so")
SOURCES = ["moe_api.cu"]
HEADERS = ["ptx_sm100.cuh", "token_kernels.cuh", "grouped_gemm_sm100.cuh", "grouped_gemm_mxf8_sm100.cuh",
           "grouped_gemm_pair_sm100.cuh", "grouped_gemm_mxf8_pair_sm100.cuh",
           "grouped_gemm_kgroup_pair_sm100.cuh", "grouped_gemm_mxf8_kgroup_pair_sm100.cuh"]
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared",
]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _inputs() -> list[str]:
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "moe_grouped.h"))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, extra_flags: list[str] | None = None) -> str:
    if not force and up_to_date():
        return LIB
    # MOE_NVCC_FLAGS: extra nvcc flags for experiments with the kernels' compile-time
    # shapes (e.g. "-DMOE_MX2_STAGES=6 -DMOE_MX2_CHUNKS=1")
    env_flags = os.environ.get("MOE_NVCC_FLAGS", "").split()
    cmd = [_nvcc(), *NVCC_FLAGS, *env_flags, *(extra_flags or []), "-I", os.path.join(ROOT, "include"),
           "-o", LIB + ".tmp", *[os.path.join(CSRC, s) for s in SOURCES]]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libmoe_grouped.so")
    if verbose and (r.stdout or r.stderr):
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true", help="print registers/spills (-Xptxas -v)")
    a = ap.parse_args()
    flags = ["-Xptxas", "-v"] if a.ptxas_info else None
    print(build(force=a.force or a.ptxas_info, verbose=a.verbose or a.ptxas_info, extra_flags=flags))
