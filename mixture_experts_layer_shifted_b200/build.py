"""Builds the in-tree shared libraries with nvcc for sm_100a.

libzcmoe.so   - the layer (C ABI in include/zcmoe.h)
libzcsynth.so - the seeded device input generator

Run as ``python -m mixture_experts_layer_shifted_b200.build`` or through
``__graft_entry__.build()``.  Rebuilds only when a source is newer than its library.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared",
          "-cudart", "shared", "-Xlinker", "-rpath,/usr/local/cuda/lib64",
          "--expt-relaxed-constexpr"]

LAYER_SOURCES = ["zcmoe.cu", "route.cu", "gemm_tc.cu", "gemm_simt.cu", "route_noalloc.cu", "fp8_quant.cu", "gemm_fp8.cu", "gemm_bwd.cu", "moe_bwd.cu", "ep.cu"]
LAYER_HEADERS = ["zc_internal.h", "zc_ptx.cuh", "zc_route.cuh", "zc_fp8.cuh"]


def _stale(target, deps):
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


def _run(cmd):
    print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)


def build(force: bool = False, verbose_ptxas: bool = False) -> None:
    layer_so = os.path.join(HERE, "libzcmoe.so")
    srcs = [os.path.join(CSRC, s) for s in LAYER_SOURCES]
    deps = srcs + [os.path.join(CSRC, h) for h in LAYER_HEADERS] + [os.path.join(ROOT, "include", "zcmoe.h")]
    if force or _stale(layer_so, deps):
        extra = ["-Xptxas", "-v"] if verbose_ptxas else []
        _run([NVCC, *ARCH, *COMMON, *extra, "-I", os.path.join(ROOT, "include"), "-o", layer_so, *srcs])
    synth_so = os.path.join(HERE, "synth", "libzcsynth.so")
    synth_src = os.path.join(HERE, "synth", "synth.cu")
    if force or _stale(synth_so, [synth_src]):
        _run([NVCC, *ARCH, *COMMON, "-o", synth_so, synth_src])


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv)
