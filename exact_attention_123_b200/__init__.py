"""Python binding for libattn, the B200 (sm_100a) fused exact-attention library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind ``include/libattn.h``.  PyTorch supplies device memory and the
current stream.  There is no CPU or library fallback: if ``libattn.so`` is
missing, importing the entry points raises.

The names follow the C ABI: ``attn_fwd``, ``attn_fwd_masked``, ``attn_fwd_varlen``,
``attn_bwd``, ``attn_bwd_deterministic``, ``attn_bwd_varlen``, ``attn_bwd_phase``, ``attn_bwd_noalloc``,
``attn_fwd_blocksparse``, ``attn_bwd_blocksparse``, ``attn_fwd_fp8``, ``attn_fwd_fp8_masked``,
``attn_fwd_fp8_varlen``, ``attn_fwd_fp8_blocksparse``,
``attn_bwd_workspace_bytes``, ``attn_bwd_deterministic_workspace_bytes``,
``attn_bwd_varlen_workspace_bytes``, ``attn_status``, ``attn_strerror``,
``attn_set_wait_limit_ms``, ``attn_debug_skip_load``, ``attn_debug_ex2_poly``, ``attn_debug_force_band``,
``attn_debug_checks``, ``attn_debug_corrupt_tag``.

With the environment variable ``LIBATTN_DEBUG=1`` at import, the binding loads
``libattn_debug.so`` instead: the same kernels with pipeline consistency checks
(``attn_debug_checks``); ``use_debug_library`` switches between the two at run time.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libattn.so")
DEBUG_LIB_PATH = os.path.join(_HERE, "libattn_debug.so")

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_MISALIGNED = 3
ATTN_ERR_WORKSPACE = 4
ATTN_ERR_CUDA = 5
ATTN_ERR_TIMEOUT = 6
ATTN_ERR_DEBUG_CHECK = 7

_lib = None
_debug = os.environ.get("LIBATTN_DEBUG", "0") not in ("", "0")
_loaded = {}


class AttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: libattn status {code}: {attn_strerror(code)}")


def use_debug_library(debug: bool) -> bool:
    """Route later calls to libattn_debug.so (True) or libattn.so (False); returns the
    previous choice.  The two libraries keep separate device state (status word,
    hooks), so a status is read from the library that ran the kernels."""
    global _lib, _debug
    prev = _debug
    _debug = bool(debug)
    _lib = None
    return prev


def lib() -> ctypes.CDLL:
    """Load libattn.so (or libattn_debug.so, see ``use_debug_library``) from the
    package directory (built by ``build.py``)."""
    global _lib
    if _lib is not None:
        return _lib
    path = DEBUG_LIB_PATH if _debug else LIB_PATH
    if path in _loaded:
        _lib = _loaded[path]
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{os.path.basename(path)} not found at {path}; build it with "
                           "`python -m exact_attention_123_b200.build` (no fallback exists)")
    L = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, vp]
    L.attn_fwd_masked.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, vp, vp]
    L.attn_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, vp, vp]
    L.attn_bwd_workspace_bytes.argtypes = [i, i, i, i]
    L.attn_bwd_workspace_bytes.restype = sz
    L.attn_bwd_varlen_workspace_bytes.argtypes = [i, i, i]
    L.attn_bwd_varlen_workspace_bytes.restype = sz
    L.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, vp, vp, sz, vp]
    L.attn_bwd_deterministic.argtypes = L.attn_bwd.argtypes
    L.attn_bwd_deterministic_workspace_bytes.argtypes = [i, i, i, i]
    L.attn_bwd_deterministic_workspace_bytes.restype = sz
    L.attn_bwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, vp, vp, sz, vp]
    L.attn_bwd_phase.argtypes = [i, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, vp, vp, sz, vp]
    L.attn_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, vp, vp]
    L.attn_fwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, vp]
    L.attn_bwd_blocksparse.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp, vp, sz, vp]
    L.attn_bwd_noalloc.restype = i
    L.attn_fwd_fp8.argtypes = [vp, vp, vp, f, f, f, vp, vp, i, i, i, i, f, i, vp]
    L.attn_fwd_fp8_masked.argtypes = [vp, vp, vp, f, f, f, vp, vp, i, i, i, i, f, i, vp, vp]
    L.attn_fwd_fp8_varlen.argtypes = [vp, vp, vp, f, f, f, vp, vp, i, i, i, i, i, f, i, vp, vp, vp]
    L.attn_fwd_fp8_blocksparse.argtypes = [vp, vp, vp, f, f, f, vp, vp, i, i, i, i, f, i, vp, vp]
    L.attn_status.argtypes = [vp]
    L.attn_strerror.argtypes = [i]
    L.attn_strerror.restype = ctypes.c_char_p
    L.attn_set_wait_limit_ms.argtypes = [i]
    L.attn_debug_skip_load.argtypes = [i]
    L.attn_debug_force_band.argtypes = [i]
    L.attn_debug_checks.argtypes = []
    L.attn_debug_corrupt_tag.argtypes = [i]
    L.attn_debug_ex2_poly.argtypes = [vp, vp, ctypes.c_longlong, vp]
    for name in ("attn_fwd", "attn_fwd_masked", "attn_fwd_varlen", "attn_bwd", "attn_bwd_deterministic",
                 "attn_bwd_varlen", "attn_bwd_phase",
                 "attn_fwd_blocksparse", "attn_bwd_blocksparse", "attn_fwd_fp8", "attn_fwd_fp8_masked",
                 "attn_fwd_fp8_varlen", "attn_fwd_fp8_blocksparse", "attn_status", "attn_set_wait_limit_ms",
                 "attn_debug_skip_load", "attn_debug_ex2_poly", "attn_debug_force_band", "attn_debug_checks",
                 "attn_debug_corrupt_tag"):
        getattr(L, name).restype = i
    _loaded[path] = L
    _lib = L
    return L


def attn_strerror(code: int) -> str:
    return lib().attn_strerror(int(code)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(rc: int, where: str):
    if rc != ATTN_OK:
        raise AttnError(rc, where)


def _need(t: torch.Tensor, dtype, name: str):
    dtypes = dtype if isinstance(dtype, tuple) else (dtype,)
    if not isinstance(t, torch.Tensor) or t.dtype not in dtypes or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA {' or '.join(str(x) for x in dtypes)} tensor")


# The library takes raw pointers and the sizes passed with them, so every tensor's
# shape and device are checked here: a buffer smaller than the sizes say would be
# read or written out of bounds on the device.
def _shaped(t, shape, dtype, name: str, device):
    _need(t, dtype, name)
    if tuple(t.shape) != tuple(shape) or t.device != device:
        raise ValueError(f"{name} must have shape {tuple(shape)} on {device}, got {tuple(t.shape)} on {t.device}")


def _inputs(tensors, dtype, packed: bool):
    """(name, tensor) pairs that must all be shaped like the first: [B,H,N,d] dense or
    [total,H,d] packed, contiguous, on one CUDA device."""
    (n0, t0), rest = tensors[0], tensors[1:]
    _need(t0, dtype, n0)
    if t0.dim() != (3 if packed else 4):
        raise ValueError(f"{n0} must be {'[total, H, d]' if packed else '[B, H, N, d]'}, got shape {tuple(t0.shape)}")
    for n, t in rest:
        _shaped(t, t0.shape, dtype, n, t0.device)
    return t0


def _side(q, cu_seqlens, key_keep, keys: int):
    """cu_seqlens: 1-D int32 on q's device; key_keep: uint8 with `keys` elements."""
    if cu_seqlens is not None:
        _need(cu_seqlens, torch.int32, "cu_seqlens")
        if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2 or cu_seqlens.device != q.device:
            raise ValueError("cu_seqlens must be a 1-D int32 tensor of B+1 offsets on q's device")
    if key_keep is not None:
        _need(key_keep, torch.uint8, "key_keep")
        if key_keep.numel() != keys or key_keep.device != q.device:
            raise ValueError(f"key_keep must hold {keys} uint8 flags on q's device, got {key_keep.numel()}")


def attn_fwd(q, k, v, o=None, lse=None, *, scale: Optional[float] = None, causal: bool = True,
             cu_seqlens: Optional[torch.Tensor] = None, key_keep: Optional[torch.Tensor] = None,
             max_seqlen: Optional[int] = None, stream=None):
    """Forward pass.  Dense q/k/v are [B,H,N,d]; packed ones are [total,H,d] with
    ``cu_seqlens`` (int32, device).  Returns (o, lse)."""
    packed = cu_seqlens is not None
    _inputs([("q", q), ("k", k), ("v", v)], torch.bfloat16, packed)
    _side(q, cu_seqlens, key_keep, q.shape[0] if packed else q.shape[0] * q.shape[2])
    d = q.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o is None:
        o = torch.empty_like(q)
    _shaped(o, q.shape, torch.bfloat16, "o", q.device)
    if cu_seqlens is not None:
        total, H = q.shape[0], q.shape[1]
        B = cu_seqlens.numel() - 1
        if lse is None:
            lse = torch.empty((total, H), device=q.device, dtype=torch.float32)
        _shaped(lse, (total, H), torch.float32, "lse", q.device)
        if max_seqlen is None:
            raise ValueError("max_seqlen is required with cu_seqlens")
        rc = lib().attn_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, total, int(max_seqlen), H, d,
                                   float(scale), int(causal), _ptr(cu_seqlens), _ptr(key_keep), _stream(stream))
        _check(rc, "attn_fwd_varlen")
        return o, lse
    B, H, N, _ = q.shape
    if lse is None:
        lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    _shaped(lse, (B, H, N), torch.float32, "lse", q.device)
    if key_keep is None:
        rc = lib().attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, float(scale), int(causal),
                            None, _stream(stream))
        _check(rc, "attn_fwd")
    else:
        rc = lib().attn_fwd_masked(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, float(scale),
                                   int(causal), None, _ptr(key_keep), _stream(stream))
        _check(rc, "attn_fwd_masked")
    return o, lse


def attn_fwd_masked(q, k, v, key_keep, **kw):
    return attn_fwd(q, k, v, key_keep=key_keep, **kw)


def attn_fwd_varlen(q, k, v, cu_seqlens, max_seqlen, **kw):
    return attn_fwd(q, k, v, cu_seqlens=cu_seqlens, max_seqlen=max_seqlen, **kw)


def attn_bwd_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(lib().attn_bwd_workspace_bytes(B, H, N, d))


def attn_bwd_deterministic_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(lib().attn_bwd_deterministic_workspace_bytes(B, H, N, d))


def attn_bwd_varlen_workspace_bytes(total: int, H: int, d: int) -> int:
    return int(lib().attn_bwd_varlen_workspace_bytes(total, H, d))


def workspace_for(q: torch.Tensor, cu_seqlens=None, deterministic: bool = False) -> torch.Tensor:
    """Allocate (with torch) a backward workspace sized for q's shape (the smaller
    one of the deterministic backward when ``deterministic``)."""
    if cu_seqlens is not None:
        if deterministic:
            n = attn_bwd_deterministic_workspace_bytes(1, q.shape[1], q.shape[0], q.shape[2])
        else:
            n = attn_bwd_varlen_workspace_bytes(q.shape[0], q.shape[1], q.shape[2])
    else:
        B, H, N, d = q.shape
        n = (attn_bwd_deterministic_workspace_bytes if deterministic else attn_bwd_workspace_bytes)(B, H, N, d)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)


def attn_bwd(q, k, v, o, lse, do, dq=None, dk=None, dv=None, *, scale: Optional[float] = None,
             causal: bool = True, cu_seqlens=None, key_keep=None, max_seqlen: Optional[int] = None,
             workspace: Optional[torch.Tensor] = None, deterministic: bool = False, stream=None):
    """Backward pass.  Returns (dq, dk, dv).  ``deterministic`` selects the
    bit-reproducible variant (``attn_bwd_deterministic``; for packed inputs its
    three phases through ``attn_bwd_phase``)."""
    packed = cu_seqlens is not None
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _inputs([("q", q), ("k", k), ("v", v), ("o", o), ("do", do), ("dq", dq), ("dk", dk), ("dv", dv)],
            torch.bfloat16, packed)
    _shaped(lse, q.shape[:2] if packed else q.shape[:3], torch.float32, "lse", q.device)
    _side(q, cu_seqlens, key_keep, q.shape[0] if packed else q.shape[0] * q.shape[2])
    d = q.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if workspace is None:
        workspace = workspace_for(q, cu_seqlens, deterministic)
    _need(workspace, torch.uint8, "workspace")
    if cu_seqlens is not None and deterministic:
        if max_seqlen is None:
            raise ValueError("max_seqlen is required with cu_seqlens")
        for ph in range(3):
            attn_bwd_phase(ph, q, k, v, o, lse, do, dq, dk, dv, workspace=workspace, scale=scale, causal=causal,
                           cu_seqlens=cu_seqlens, key_keep=key_keep, max_seqlen=max_seqlen, stream=stream)
    elif cu_seqlens is not None:
        total, H = q.shape[0], q.shape[1]
        B = cu_seqlens.numel() - 1
        if max_seqlen is None:
            raise ValueError("max_seqlen is required with cu_seqlens")
        rc = lib().attn_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk),
                                   _ptr(dv), B, total, int(max_seqlen), H, d, float(scale), int(causal),
                                   _ptr(cu_seqlens), _ptr(key_keep), _ptr(workspace), workspace.numel(),
                                   _stream(stream))
        _check(rc, "attn_bwd_varlen")
    else:
        B, H, N, _ = q.shape
        name = "attn_bwd_deterministic" if deterministic else "attn_bwd"
        rc = getattr(lib(), name)(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk),
                                  _ptr(dv), B, H, N, d, float(scale), int(causal), None, _ptr(key_keep),
                                  _ptr(workspace), workspace.numel(), _stream(stream))
        _check(rc, name)
    return dq, dk, dv


def attn_fwd_blocksparse(q, k, v, block_mask, o=None, lse=None, *, scale: Optional[float] = None,
                         causal: bool = False, stream=None):
    """Block-sparse forward (dense [B,H,N,d] layout).  block_mask: uint8 device tensor
    [H, ceil(N/128), ceil(N/128)]; a zero leaves that (query tile, key tile) pair out.
    Returns (o, lse)."""
    _inputs([("q", q), ("k", k), ("v", v)], torch.bfloat16, False)
    B, H, N, d = q.shape
    nb = (N + 127) // 128
    _shaped(block_mask, (H, nb, nb), torch.uint8, "block_mask", q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32) if lse is None else lse
    _shaped(o, q.shape, torch.bfloat16, "o", q.device)
    _shaped(lse, (B, H, N), torch.float32, "lse", q.device)
    rc = lib().attn_fwd_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, float(scale),
                                    int(causal), _ptr(block_mask), _stream(stream))
    _check(rc, "attn_fwd_blocksparse")
    return o, lse


def attn_bwd_blocksparse(q, k, v, o, lse, do, block_mask, dq=None, dk=None, dv=None, *,
                         scale: Optional[float] = None, causal: bool = False,
                         workspace: Optional[torch.Tensor] = None, stream=None):
    """Block-sparse backward (dense layout, same block_mask as the forward).
    Returns (dq, dk, dv)."""
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _inputs([("q", q), ("k", k), ("v", v), ("o", o), ("do", do), ("dq", dq), ("dk", dk), ("dv", dv)],
            torch.bfloat16, False)
    B, H, N, d = q.shape
    nb = (N + 127) // 128
    _shaped(lse, (B, H, N), torch.float32, "lse", q.device)
    _shaped(block_mask, (H, nb, nb), torch.uint8, "block_mask", q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if workspace is None:
        workspace = workspace_for(q)
    _need(workspace, torch.uint8, "workspace")
    rc = lib().attn_bwd_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk),
                                    _ptr(dv), B, H, N, d, float(scale), int(causal), _ptr(block_mask),
                                    _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "attn_bwd_blocksparse")
    return dq, dk, dv


def attn_fwd_fp8(q, k, v, q_scale: float, k_scale: float, v_scale: float, o=None, lse=None, *,
                 scale: Optional[float] = None, causal: bool = True, cu_seqlens: Optional[torch.Tensor] = None,
                 key_keep: Optional[torch.Tensor] = None, max_seqlen: Optional[int] = None, stream=None):
    """FP8 forward.  q, k, v: e4m3 codes (torch.float8_e4m3fn, or uint8 views of them)
    whose values are code * {q,k,v}_scale, dense [B,H,N,d] or packed [total,H,d] with
    ``cu_seqlens`` (int32, device) and ``max_seqlen``; optional per-key ``key_keep``.
    Returns (o bf16, lse fp32)."""
    codes = (torch.float8_e4m3fn, torch.uint8)
    packed = cu_seqlens is not None
    _inputs([("q", q), ("k", k), ("v", v)], codes, packed)
    _side(q, cu_seqlens, key_keep, q.shape[0] if packed else q.shape[0] * q.shape[2])
    d = q.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = torch.empty(q.shape, device=q.device, dtype=torch.bfloat16) if o is None else o
    _shaped(o, q.shape, torch.bfloat16, "o", q.device)
    lse_shape = q.shape[:2] if packed else q.shape[:3]
    lse = torch.empty(lse_shape, device=q.device, dtype=torch.float32) if lse is None else lse
    _shaped(lse, lse_shape, torch.float32, "lse", q.device)
    sc = (float(q_scale), float(k_scale), float(v_scale))
    if packed:
        if max_seqlen is None:
            raise ValueError("max_seqlen is required with cu_seqlens")
        total, H = q.shape[0], q.shape[1]
        rc = lib().attn_fwd_fp8_varlen(_ptr(q), _ptr(k), _ptr(v), *sc, _ptr(o), _ptr(lse), cu_seqlens.numel() - 1,
                                       total, int(max_seqlen), H, d, float(scale), int(causal), _ptr(cu_seqlens),
                                       _ptr(key_keep), _stream(stream))
        _check(rc, "attn_fwd_fp8_varlen")
        return o, lse
    B, H, N, _ = q.shape
    if key_keep is None:
        rc = lib().attn_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), *sc, _ptr(o), _ptr(lse), B, H, N, d, float(scale),
                                int(causal), _stream(stream))
        _check(rc, "attn_fwd_fp8")
    else:
        rc = lib().attn_fwd_fp8_masked(_ptr(q), _ptr(k), _ptr(v), *sc, _ptr(o), _ptr(lse), B, H, N, d, float(scale),
                                       int(causal), _ptr(key_keep), _stream(stream))
        _check(rc, "attn_fwd_fp8_masked")
    return o, lse


def attn_fwd_fp8_blocksparse(q, k, v, q_scale: float, k_scale: float, v_scale: float, block_mask, o=None, lse=None,
                             *, scale: Optional[float] = None, causal: bool = True, stream=None):
    """FP8 forward with a tile mask.  q, k, v: e4m3 codes (torch.float8_e4m3fn, or uint8
    views of them) [B,H,N,d] whose values are code * {q,k,v}_scale; block_mask: uint8
    device tensor [H, ceil(N/128), ceil(N/128)] as for ``attn_fwd_blocksparse``.
    Returns (o bf16, lse fp32)."""
    _inputs([("q", q), ("k", k), ("v", v)], (torch.float8_e4m3fn, torch.uint8), False)
    B, H, N, d = q.shape
    nb = (N + 127) // 128
    _shaped(block_mask, (H, nb, nb), torch.uint8, "block_mask", q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = torch.empty(q.shape, device=q.device, dtype=torch.bfloat16) if o is None else o
    lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32) if lse is None else lse
    _shaped(o, q.shape, torch.bfloat16, "o", q.device)
    _shaped(lse, (B, H, N), torch.float32, "lse", q.device)
    rc = lib().attn_fwd_fp8_blocksparse(_ptr(q), _ptr(k), _ptr(v), float(q_scale), float(k_scale), float(v_scale),
                                        _ptr(o), _ptr(lse), B, H, N, d, float(scale), int(causal), _ptr(block_mask),
                                        _stream(stream))
    _check(rc, "attn_fwd_fp8_blocksparse")
    return o, lse


def attn_bwd_deterministic(q, k, v, o, lse, do, dq=None, dk=None, dv=None, **kw):
    """attn_bwd with bit-reproducible results (dK/dV and dQ in separate passes)."""
    return attn_bwd(q, k, v, o, lse, do, dq, dk, dv, deterministic=True, **kw)


def attn_bwd_phase(phase: int, q, k, v, o, lse, do, dq, dk, dv, *, workspace, scale: Optional[float] = None,
                   causal: bool = True, cu_seqlens=None, key_keep=None, max_seqlen: Optional[int] = None,
                   stream=None):
    """Launch one backward phase (0 preprocess, 1 dK/dV, 2 dQ)."""
    packed = cu_seqlens is not None
    _inputs([("q", q), ("k", k), ("v", v), ("o", o), ("do", do), ("dq", dq), ("dk", dk), ("dv", dv)],
            torch.bfloat16, packed)
    _shaped(lse, q.shape[:2] if packed else q.shape[:3], torch.float32, "lse", q.device)
    _side(q, cu_seqlens, key_keep, q.shape[0] if packed else q.shape[0] * q.shape[2])
    _need(workspace, torch.uint8, "workspace")
    d = q.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if cu_seqlens is not None:
        nseq, total, H, N = cu_seqlens.numel() - 1, q.shape[0], q.shape[1], int(max_seqlen)
    else:
        nseq, H, N, _ = q.shape
        total = 0
    rc = lib().attn_bwd_phase(int(phase), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq),
                              _ptr(dk), _ptr(dv), nseq, total, N, H, d, float(scale), int(causal), _ptr(cu_seqlens),
                              _ptr(key_keep), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(rc, "attn_bwd_phase")


def attn_bwd_noalloc(q, k, v, o, lse, do, dq=None, dk=None, dv=None, *, scale: Optional[float] = None,
                     causal: bool = True, key_keep=None, stream=None):
    """Dense-layout backward that uses the library's own scratch array instead of a
    caller workspace, for callers that cannot allocate device memory (see the C
    declaration for the size limit and the sharing rules).  Returns (dq, dk, dv)."""
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    _inputs([("q", q), ("k", k), ("v", v), ("o", o), ("do", do), ("dq", dq), ("dk", dk), ("dv", dv)],
            torch.bfloat16, False)
    _shaped(lse, q.shape[:3], torch.float32, "lse", q.device)
    _side(q, None, key_keep, q.shape[0] * q.shape[2])
    B, H, N, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    rc = lib().attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk),
                                _ptr(dv), B, H, N, d, float(scale), int(causal), None, _ptr(key_keep),
                                _stream(stream))
    _check(rc, "attn_bwd_noalloc")
    return dq, dk, dv


def attn_status(stream=None) -> int:
    """Synchronise the stream; return and clear the device status word."""
    return int(lib().attn_status(_stream(stream)))


def attn_set_wait_limit_ms(ms: int) -> int:
    return int(lib().attn_set_wait_limit_ms(int(ms)))


def attn_debug_skip_load(index: int) -> int:
    return int(lib().attn_debug_skip_load(int(index)))


def attn_debug_force_band(slices: int) -> int:
    """Test hook: force bands of `slices` slices in the banded unit order (0: automatic).
    Returns the previous value."""
    return int(lib().attn_debug_force_band(int(slices)))


def attn_debug_checks() -> bool:
    """True when the loaded library is the debug build (pipeline consistency checks)."""
    return bool(lib().attn_debug_checks())


def attn_debug_corrupt_tag(fill_index: int) -> int:
    """Test hook (debug library): the forward producer writes a wrong check tag for ring
    fill `fill_index` of each CTA (-1: off).  Returns the previous value."""
    return int(lib().attn_debug_corrupt_tag(int(fill_index)))


def attn_debug_ex2_poly(x: torch.Tensor, stream=None) -> torch.Tensor:
    """The forward kernels' FMA-pipe 2^x on a float32 CUDA tensor of even size
    (test hook).  Returns y of x's shape."""
    _need(x, torch.float32, "x")
    y = torch.empty_like(x)
    _check(lib().attn_debug_ex2_poly(_ptr(x), _ptr(y), x.numel(), _stream(stream)), "attn_debug_ex2_poly")
    return y
