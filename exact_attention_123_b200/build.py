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
# the same kernels with pipeline consistency checks (LIBATTN_DEBUG=1; see attn_debug_checks)
LIB_DEBUG = os.path.join(HERE, "libattn_debug.so")
SOURCES = ["attn_api.cu", "attn_fwd_sm100.cu", "attn_bwd_sm100.cu", "attn_bwd_fused_sm100.cu", "attn_noalloc.cu"]
HEADERS = ["sm100_ptx.cuh", "attn_common.cuh", "attn_launch.h", "../../include/libattn.h"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.abspath(__file__)]
    return any(os.path.getmtime(p) > t for p in deps if os.path.exists(p))


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Builds libattn.so and (debug=True) libattn_debug.so, each only if stale or
    forced, the two compilations side by side.  Returns the release library's path."""
    flags = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
             "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
             "-shared", "-cudart", "static"]
    if verbose:
        flags += ["-Xptxas", "-v"]
    srcs = [os.path.join(CSRC, f) for f in SOURCES]
    jobs = []
    for lib, extra in ((LIB, []), (LIB_DEBUG, ["-DLIBATTN_DEBUG=1"])):
        if (lib == LIB_DEBUG and not debug) or not (force or _stale(lib)):
            continue
        jobs.append((lib, subprocess.Popen([nvcc()] + flags + extra + srcs + ["-o", lib + ".tmp"])))
    failed = [lib for lib, proc in jobs if proc.wait() != 0]
    if failed:
        raise subprocess.CalledProcessError(1, f"nvcc ({', '.join(os.path.basename(f) for f in failed)})")
    for lib, _ in jobs:
        os.replace(lib + ".tmp", lib)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
