"""Build the CUDA library of the package (sm_100a) in place.

    python -m mixture_experts_ffn_05_b200.build

Produces mixture_experts_ffn_05_b200/libmoeffn.so from csrc/*.cu with nvcc.  The CUDA
runtime is linked statically; the driver's tensor-map encoder is looked up at run
time, so the library loads on a machine without a GPU (only its compute calls need
one).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SOURCES = ["router.cu", "router_tc.cu", "permute.cu", "grouped_gemm.cu", "stream_gemm.cu",
           "combine.cu", "quant.cu", "health.cu", "moe_ffn.cu"]
LIB = os.path.join(PKG, "libmoeffn.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if c and os.path.exists(c):
            return c
    raise RuntimeError("nvcc not found")


def build(verbose: bool = False, force: bool = False) -> str:
    srcs = [os.path.join(PKG, "csrc", s) for s in SOURCES]
    deps = srcs + [os.path.join(PKG, "csrc", h) for h in ("common.cuh", "internal.h", "permute_impl.cuh", "warp_mma.cuh")] + [
        os.path.join(ROOT, "include", "moe_ffn.h")]
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(d) <= t for d in deps):
            return LIB
    tmp = LIB + ".tmp"
    cmd = [nvcc(), *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-I" + os.path.join(ROOT, "include"), "-o", tmp, *srcs]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(verbose="-v" in sys.argv, force="-f" in sys.argv))
