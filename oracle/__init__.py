"""CPU float64 attention oracle -- TEST INFRASTRUCTURE.

Only ``tests/``, the smoke check in ``__graft_entry__`` and the CPU-baseline leg
of ``bench.py`` may import this package.  The CUDA library never calls it and
there is no fallback from the product path into it.

``fwd`` / ``bwd`` wrap the C implementation in ``attn_oracle.c`` (plain float64,
OpenMP over rows, no BLAS).  Inputs are upcast exactly from bf16 to float64.
``e4m3_decode`` / ``fwd_fp8`` give the attention of 8-bit e4m3 inputs: the codes are
decoded exactly to float64 (times their per-tensor factor), then ``fwd`` runs.
See ``attn_oracle.c`` for the definition and the passages it follows.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        up = ctypes.POINTER(ctypes.c_ubyte)
        L.oracle_attn_fwd.argtypes = [dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_double, ctypes.c_int, ip, up, up, ctypes.c_int,
                                      ip, ctypes.c_int, ctypes.c_int]
        L.oracle_attn_fwd.restype = ctypes.c_int
        L.oracle_attn_bwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int,
                                      ip, up, up, ctypes.c_int, ip, ctypes.c_int, ctypes.c_int]
        L.oracle_attn_bwd.restype = ctypes.c_int
        L.oracle_max_threads.restype = ctypes.c_int
        L.oracle_e4m3_decode.argtypes = [up, ctypes.c_long, ctypes.c_double, dp]
        L.oracle_e4m3_decode.restype = None
        _lib = L
    return _lib


def _f64(x):
    """Exact upcast of a torch tensor or array-like to a C-contiguous float64 array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().cpu().to(torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x):
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _u8(x):
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.uint8))


def _ptr(a, ct):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ct))


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def fwd(q, k, v, scale, causal, cu_seqlens=None, key_keep=None, slices=None, nthreads=None, N=None,
        block_mask=None, block=128):
    """Forward pass.  q,k,v: dense [B,H,N,d] or packed [total,H,d] (with cu_seqlens).

    block_mask (dense layout only): [H, ceil(N/block), ceil(N/block)] uint8 tile mask;
    a zero leaves the whole (query tile, key tile) pair out.

    Returns (o, lse) as float64 arrays with the input's layout ([B,H,N] / [total,H] for lse).
    Rows of slices not listed in ``slices`` (b*H+h indices) are left as NaN.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    cu = _i32(cu_seqlens)
    kk = _u8(key_keep)
    if cu is None:
        B, H, Nn, d = q.shape
        lse = np.full((B, H, Nn), np.nan)
    else:
        _, H, d = q.shape
        B = len(cu) - 1
        Nn = int(N if N is not None else max(int(cu[i + 1] - cu[i]) for i in range(B)))
        lse = np.full((q.shape[0], H), np.nan)
    o = np.full(q.shape, np.nan)
    sl = _i32(slices)
    bm = _u8(block_mask)
    rc = lib().oracle_attn_fwd(_ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double), _ptr(v, ctypes.c_double),
                               _ptr(o, ctypes.c_double), _ptr(lse, ctypes.c_double), B, H, Nn, d,
                               float(scale), int(bool(causal)), _ptr(cu, ctypes.c_int), _ptr(kk, ctypes.c_ubyte),
                               _ptr(bm, ctypes.c_ubyte), int(block),
                               _ptr(sl, ctypes.c_int), 0 if sl is None else len(sl),
                               int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError("oracle_attn_fwd rejected its arguments")
    return o, lse


def bwd(q, k, v, dout, scale, causal, cu_seqlens=None, key_keep=None, slices=None, nthreads=None, N=None,
        block_mask=None, block=128):
    """Backward pass from the softmax Jacobian.  Returns (dq, dk, dv) float64."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    cu = _i32(cu_seqlens)
    kk = _u8(key_keep)
    if cu is None:
        B, H, Nn, d = q.shape
    else:
        _, H, d = q.shape
        B = len(cu) - 1
        Nn = int(N if N is not None else max(int(cu[i + 1] - cu[i]) for i in range(B)))
    dq = np.full(q.shape, np.nan)
    dk = np.full(q.shape, np.nan)
    dv = np.full(q.shape, np.nan)
    sl = _i32(slices)
    bm = _u8(block_mask)
    rc = lib().oracle_attn_bwd(_ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double), _ptr(v, ctypes.c_double),
                               _ptr(dout, ctypes.c_double), _ptr(dq, ctypes.c_double),
                               _ptr(dk, ctypes.c_double), _ptr(dv, ctypes.c_double), B, H, Nn, d,
                               float(scale), int(bool(causal)), _ptr(cu, ctypes.c_int), _ptr(kk, ctypes.c_ubyte),
                               _ptr(bm, ctypes.c_ubyte), int(block),
                               _ptr(sl, ctypes.c_int), 0 if sl is None else len(sl),
                               int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError("oracle_attn_bwd rejected its arguments")
    return dq, dk, dv


def e4m3_decode(codes, factor=1.0):
    """float64 values of e4m3 codes (uint8 array-like or a torch float8_e4m3fn / uint8
    tensor) times ``factor``; same shape."""
    try:
        import torch
        if isinstance(codes, torch.Tensor):
            codes = codes.detach().cpu()
            if codes.dtype != torch.uint8:
                codes = codes.view(torch.uint8)
            codes = codes.numpy()
    except ImportError:  # pragma: no cover
        pass
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.uint8))
    out = np.empty(c.shape, dtype=np.float64)
    lib().oracle_e4m3_decode(_ptr(c, ctypes.c_ubyte), c.size, float(factor), _ptr(out, ctypes.c_double))
    return out


def fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, scale, causal, cu_seqlens=None, key_keep=None, slices=None,
            nthreads=None, N=None, block_mask=None):
    """Forward of e4m3 inputs (dense [B,H,N,d] or packed [total,H,d] with cu_seqlens):
    the attention of the decoded values (code value x per-tensor factor), with the
    same masks as ``fwd`` (the tile mask included).  Returns (o, lse) float64 like
    ``fwd``."""
    return fwd(e4m3_decode(q8, q_scale), e4m3_decode(k8, k_scale), e4m3_decode(v8, v_scale), scale, causal,
               cu_seqlens=cu_seqlens, key_keep=key_keep, slices=slices, nthreads=nthreads, N=N,
               block_mask=block_mask)

