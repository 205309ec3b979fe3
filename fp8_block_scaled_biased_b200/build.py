"""Build libfp8moe.so (sm_100a) in-tree with nvcc.

    python -m fp8_block_scaled_biased_b200.build [--verbose]

The library is one translation unit (csrc/fp8moe.cu) compiled for
sm_100a only, position-independent, linked against the CUDA runtime. No
libcuda link is needed: the TMA tensor-map encoder is fetched at run time
through cudaGetDriverEntryPoint.
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
SRC = os.path.join(PKG_DIR, "csrc", "fp8moe.cu")
LIB = os.path.join(PKG_DIR, "libfp8moe.so")
DEPS = [os.path.join(PKG_DIR, "csrc", f) for f in sorted(os.listdir(os.path.join(PKG_DIR, "csrc")))]
DEPS.append(os.path.join(ROOT, "include", "fp8moe.h"))


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def command(verbose: bool = False, out: str = LIB) -> list[str]:
    cmd = [
        nvcc_path(), "-std=c++17", "-O3", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-Xcompiler", "-fPIC", "-shared",
        "-I", os.path.join(ROOT, "include"),
        "-o", out, SRC, "-lcudart",
    ]
    if verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS if os.path.exists(d))


def build(force: bool = False, verbose: bool = False) -> str:
    if force or not up_to_date():
        tmp = LIB + ".tmp"
        subprocess.run(command(verbose, tmp), check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true", help="print ptxas register/shared-memory usage")
    ap.add_argument("--force", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force or args.verbose, verbose=args.verbose))
    sys.exit(0)
