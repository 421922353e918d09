"""attn_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers may not call cudaMalloc: code that runs with a fixed memory budget,
inside another framework's allocator that forbids raw device allocations, or code
that must not allocate once it has started.  attn_bwd_noalloc serves them by using
a fixed scratch array inside the library instead of a caller-provided workspace.

This file is collected last (after every other test) on purpose.  It checks,
through the C ABI, that two calls in a row give the same gradients as attn_bwd
with a caller workspace, within the backward tolerance the other tests use, and
that sizes beyond the array are refused without any GPU work.
"""
import ctypes

import numpy as np
import pytest
import torch

from attn_inputs import make_dense

pytestmark = pytest.mark.gpu

G_ATOL, G_RTOL = 2e-2, 2e-2


@pytest.fixture(scope="module")
def ea():
    from exact_attention_123_b200 import build
    build.build()
    import exact_attention_123_b200 as m
    assert torch.cuda.is_available()
    return m


def _vp(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _close(got, ref, what):
    g = got.detach().double().cpu().numpy()
    r = ref.detach().double().cpu().numpy()
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    bad = np.abs(g - r) > G_ATOL + G_RTOL * np.abs(r)
    assert not bad.any(), f"{what}: {bad.sum()} elements differ from attn_bwd beyond tolerance"


def test_noalloc_matches_workspace_backward_on_two_calls(ea):
    inp = make_dense(2, 4, 700, 128, seed=8100, causal=True, with_grad=True)
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))
    o, lse = ea.attn_fwd(q, k, v, scale=inp.scale, causal=True)
    ref = ea.attn_bwd(q, k, v, o, lse, do, scale=inp.scale, causal=True)  # caller workspace
    assert ea.attn_status() == ea.ATTN_OK
    L = ea.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    B, H, N, d = q.shape
    for call in range(2):
        dq, dk, dv = (torch.full_like(t, float("nan")) for t in (q, k, v))
        rc = L.attn_bwd_noalloc(_vp(q), _vp(k), _vp(v), _vp(o), _vp(lse), _vp(do), _vp(dq), _vp(dk), _vp(dv),
                                B, H, N, d, ctypes.c_float(inp.scale), 1, None, None, stream)
        assert rc == ea.ATTN_OK, ea.attn_strerror(rc)
        assert ea.attn_status() == ea.ATTN_OK
        for got, want, name in zip((dq, dk, dv), ref, ("dQ", "dK", "dV")):
            _close(got, want, f"call {call + 1} {name}")


def test_noalloc_refuses_sizes_beyond_its_array(ea):
    small = torch.zeros(1, 1, 16, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 1, 16, device="cuda")
    L = ea.lib()
    # B*H*N = 4 * 64 * 8192 rows need 2 * 8 MiB of scratch: more than the array holds.
    # The size is checked before anything is launched, so the small buffers are never read.
    rc = L.attn_bwd_noalloc(_vp(small), _vp(small), _vp(small), _vp(small), _vp(lse), _vp(small), _vp(small),
                            _vp(small), _vp(small), 4, 64, 8192, 128, ctypes.c_float(0.088), 1, None, None,
                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == ea.ATTN_ERR_WORKSPACE
    assert ea.attn_bwd_workspace_bytes(4, 64, 8192, 128) > 8 * 1024 * 1024
