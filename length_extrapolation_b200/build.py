"""Build the in-tree CUDA library ``libdca_b200.so`` for sm_100a with nvcc.

Usage: ``python -m length_extrapolation_b200.build [--force] [--verbose]``.
The library is built in place (next to this file) so that it ships with the
source tree; it links the CUDA runtime statically and resolves the driver's
tensor-map encoder at run time, so it loads on machines without a GPU.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libdca_b200.so")
SOURCES = ["dca_api.cu", "dca_prep.cu", "dca_fwd_sm100.cu", "dca_fwd_f32.cu", "dca_decode_sm100.cu",
           "dca_sparse_sm100.cu", "dca_sparse_prep.cu", "dca_select.cu", "dca_select_mma.cu",
           "dca_noalloc.cu"]
HEADERS = ["dca_internal.h", "dca_plan.cuh", "dca_select_rows.cuh", "dca_softmax.cuh",
           "dca_sparse_plan.cuh",
           "sm100_ptx.cuh"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA library cannot be built")


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(os.path.dirname(HERE), "include", "dca.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    nvcc = nvcc_path()
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc, "-O3", "-std=c++17", *ARCH, "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
           "-o", tmp, *[os.path.join(CSRC, s) for s in SOURCES]]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libdca_b200.so")
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
