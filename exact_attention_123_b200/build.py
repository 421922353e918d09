"""Builds libattn.so (the sm_100a CUDA library behind include/libattn.h) in-tree.

``python -m exact_attention_123_b200.build`` or ``build()`` from Python.  The
library is compiled for sm_100a only; it statically links the CUDA runtime and
reaches the driver's tensor-map encoder through the runtime's entry-point query,
so it needs no libcuda at link time.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libattn.so")
SOURCES = ["attn_api.cu", "attn_fwd_sm100.cu", "attn_bwd_sm100.cu", "attn_bwd_fused_sm100.cu", "attn_noalloc.cu"]
HEADERS = ["sm100_ptx.cuh", "attn_common.cuh", "attn_launch.h", "../../include/libattn.h"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.abspath(__file__)]
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    flags = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
             "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
             "-shared", "-cudart", "static"]
    if verbose:
        flags += ["-Xptxas", "-v"]
    srcs = [os.path.join(CSRC, f) for f in SOURCES]
    tmp = LIB + ".tmp"
    subprocess.run([nvcc()] + flags + srcs + ["-o", tmp], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
