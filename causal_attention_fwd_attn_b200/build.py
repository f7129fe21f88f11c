"""Builds libforge_attn.so (the CUDA library behind include/forge_attn.h) in-tree.

    python -m causal_attention_fwd_attn_b200.build [--verbose]

nvcc compiles for sm_100a only (tcgen05 and TMA need the arch-specific target);
no GPU is needed to build.  ``--ptxas-info`` adds ``-Xptxas -v`` (registers,
spills and shared memory per kernel).
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
INCLUDE = os.path.join(ROOT, "include")
LIBRARY = os.path.join(PKG, "libforge_attn.so")
SOURCES = ["forge_attn_api.cu", "attn_fwd.cu", "attn_bwd.cu", "tc_probe.cu", "forge_attn_noalloc.cu",
           "adamw.cu", "gemm.cu", "convert.cu"]
HEADERS = ["sm100_ptx.cuh", "forge_internal.h"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _inputs():
    files = [os.path.join(CSRC, s) for s in SOURCES + HEADERS]
    files += [os.path.join(INCLUDE, h) for h in ("forge_attn.h", "forge_attn_testing.h", "forge_adamw.h",
                                                        "forge_linear.h")]
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIBRARY):
        return False
    t = os.path.getmtime(LIBRARY)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, ptxas_info: bool = False, verbose: bool = False) -> str:
    if not force and not ptxas_info and up_to_date():
        return LIBRARY
    # No relocatable device code: ptxas then honours per-warpgroup register budgets
    # (setmaxnreg), which the dK/dV kernel relies on.
    cmd = [nvcc_path(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared",
           "-Xcompiler", "-fPIC", "-I", INCLUDE, "-o", LIBRARY + ".tmp"]
    if ptxas_info:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed")
    if ptxas_info or verbose:
        sys.stderr.write(res.stderr)
    os.replace(LIBRARY + ".tmp", LIBRARY)
    return LIBRARY


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    a = ap.parse_args()
    print(build(force=True, ptxas_info=a.ptxas_info, verbose=a.verbose))


if __name__ == "__main__":
    main()
