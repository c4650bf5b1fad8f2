"""Build libcutbce.so in-tree with nvcc for sm_100a (B200).

Usage: python -m vocabulary_label_bce_b200.build [--force]
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libcutbce.so")
SOURCES = ["cutbce_api.cu"]
DEPS = ["cutbce_api.cu", "common.cuh", "prep_finish.cuh", "pair_sort.cuh", "tile_engine.cuh", "ptx_sm100.cuh", "probes.cuh",
        "elementwise.cuh", "topk.cuh"]


def nvcc_path() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def command(out: str = LIB, extra: list[str] | None = None) -> list[str]:
    return [nvcc_path(), "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
            "-Xcompiler", "-fPIC,-O3", "-shared", "-cudart", "static", f"-I{INCLUDE}", f"-I{CSRC}",
            "-o", out] + [os.path.join(CSRC, s) for s in SOURCES] + (extra or [])


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    srcs = [os.path.join(CSRC, d) for d in DEPS] + [os.path.join(INCLUDE, "cutbce.h")]
    return all(os.path.getmtime(s) <= t for s in srcs)


def build(force: bool = False, verbose: bool = True) -> str:
    if not force and up_to_date():
        return LIB
    cmd = command()
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv)
