"""Build the CUDA library (libdsa.so) in-tree for sm_100a.

    python -m sparse_attention_long_fp8_b200.build [--force] [--ptxas-info]

nvcc cross-compiles without a GPU; the shared object lands next to this file
so it travels with the source tree.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libdsa.so")
MAIN = os.path.join(CSRC, "dsa_api.cu")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _sources():
    inc = os.path.join(os.path.dirname(PKG), "include", "dsa.h")
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC))
            if f.endswith((".cu", ".cuh"))] + [inc]


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(s) > t for s in _sources())


def build(force: bool = False, ptxas_info: bool = False, extra=()) -> str:
    if not force and not needs_build():
        return LIB
    cuda_home = os.path.dirname(os.path.dirname(_nvcc()))
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "--expt-relaxed-constexpr",
           "-Xcompiler", "-fPIC", "-shared", "-cudart", "shared",
           "-Xlinker", f"-rpath,{cuda_home}/lib64",
           "-o", tmp, MAIN, *extra]
    if ptxas_info:
        cmd += ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True, cwd=CSRC)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, ptxas_info="--ptxas-info" in sys.argv)
    print(LIB)
