"""attn_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some callers may not call cudaMalloc: code that runs with a fixed memory budget,
inside another framework's allocator that forbids raw device allocations, or code
that must not allocate once it has started.  attn_bwd_noalloc serves them by using
a fixed scratch array inside the library instead of a caller-provided workspace.

This file is collected last (after every other test) on purpose.  Through the C
ABI it checks that two calls in a row give bit for bit the gradients of
attn_bwd_deterministic with a caller workspace (the same kernels, no atomics),
after a first call of another shape and other inputs has left different values
in the shared array; that one of them matches the float64 oracle; and that sizes
past the array are refused without any GPU work.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from attn_inputs import make_dense

pytestmark = pytest.mark.gpu

G_ATOL, G_RTOL = 2e-2, 2e-2
SCRATCH_BYTES = 8 << 20  # ATTN_NOALLOC_SCRATCH_BYTES


@pytest.fixture(scope="module")
def ea():
    from exact_attention_123_b200 import build
    build.build()
    import exact_attention_123_b200 as m
    assert torch.cuda.is_available()
    return m


def _vp(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _noalloc(ea, q, k, v, o, lse, do, scale, causal):
    L = ea.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    B, H, N, d = q.shape
    dq, dk, dv = (torch.full_like(t, float("nan")) for t in (q, k, v))
    rc = L.attn_bwd_noalloc(_vp(q), _vp(k), _vp(v), _vp(o), _vp(lse), _vp(do), _vp(dq), _vp(dk), _vp(dv),
                            B, H, N, d, ctypes.c_float(scale), int(causal), None, None, stream)
    assert rc == ea.ATTN_OK, ea.attn_strerror(rc)
    assert ea.attn_status() == ea.ATTN_OK
    return dq, dk, dv


def test_noalloc_matches_workspace_backward_on_two_calls(ea):
    # First a larger, non-causal call with other inputs: it leaves its own D and lse2
    # terms all over the shared array, so the checked calls below cannot pass by
    # reading values that happen to be right already.
    big = make_dense(3, 5, 900, 128, seed=8101, causal=False, with_grad=True)
    bq, bk, bv, bdo = (t.cuda() for t in (big.q, big.k, big.v, big.do))
    bo, blse = ea.attn_fwd(bq, bk, bv, scale=big.scale, causal=False)
    _noalloc(ea, bq, bk, bv, bo, blse, bdo, big.scale, False)

    inp = make_dense(2, 4, 700, 128, seed=8100, causal=True, with_grad=True)
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))
    o, lse = ea.attn_fwd(q, k, v, scale=inp.scale, causal=True)
    ref = ea.attn_bwd_deterministic(q, k, v, o, lse, do, scale=inp.scale, causal=True)  # caller workspace
    assert ea.attn_status() == ea.ATTN_OK
    for call in range(2):
        got = _noalloc(ea, q, k, v, o, lse, do, inp.scale, True)
        for g, want, name in zip(got, ref, ("dQ", "dK", "dV")):
            assert torch.equal(g, want), f"call {call + 1} {name} differs from attn_bwd_deterministic"
    # and the result is the right one, within the backward tolerance of the other tests
    orq, ork, orv = oracle.bwd(inp.q, inp.k, inp.v, inp.do, inp.scale, True)
    for g, r, name in zip(got, (orq, ork, orv), ("dQ", "dK", "dV")):
        x = g.double().cpu().numpy()
        assert np.all(np.isfinite(x)), name
        bad = np.abs(x - r) > G_ATOL + G_RTOL * np.abs(r)
        assert not bad.any(), f"{name}: {bad.sum()} elements differ from the oracle"


def test_noalloc_refuses_sizes_beyond_its_array(ea):
    small = torch.zeros(1, 1, 16, 128, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 1, 16, device="cuda")
    L = ea.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # The exact edge: 1,048,576 query rows x heads fill the array, one more does not fit.
    assert ea.attn_bwd_deterministic_workspace_bytes(1, 1, 1048576, 128) <= SCRATCH_BYTES
    assert ea.attn_bwd_deterministic_workspace_bytes(1, 1, 1048577, 128) > SCRATCH_BYTES
    # The size is checked before anything is launched, so the small buffers are never read.
    for shape in ((1, 1, 1048577, 128), (4, 64, 8192, 128)):
        rc = L.attn_bwd_noalloc(_vp(small), _vp(small), _vp(small), _vp(small), _vp(lse), _vp(small), _vp(small),
                                _vp(small), _vp(small), *shape, ctypes.c_float(0.088), 1, None, None, stream)
        assert rc == ea.ATTN_ERR_WORKSPACE, shape
    assert ea.attn_status() == ea.ATTN_OK
