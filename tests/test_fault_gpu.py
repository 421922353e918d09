"""Failure detection without a GPU fault.

The loader is told (through a test hook) to skip one pipeline load, so the slot
it would have filled never fills.  The consumer's bounded wait expires after the
short limit set here, every role of the kernel stops cleanly, and the host reads
ATTN_ERR_TIMEOUT from attn_status().  The context stays usable: the next call
succeeds and matches the oracle.  Nothing traps, faults or waits forever.
"""
import numpy as np
import pytest
import torch

import oracle
from attn_inputs import make_dense

pytestmark = pytest.mark.gpu


def _within(got, ref, atol, rtol):
    g = got.double().cpu().numpy()
    return np.all(np.isfinite(g)) and not (np.abs(g - ref) > atol + rtol * np.abs(ref)).any()


@pytest.fixture(scope="module")
def ea():
    from exact_attention_123_b200 import build
    build.build()
    import exact_attention_123_b200 as m
    return m


@pytest.mark.parametrize("skip", [0, 1, 3])
def test_expired_wait_reports_timeout_and_context_survives(ea, skip):
    inp = make_dense(1, 2, 384, 128, seed=7000)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    assert ea.attn_status() == ea.ATTN_OK
    prev_limit = ea.attn_set_wait_limit_ms(200)
    ea.attn_debug_skip_load(skip)
    try:
        ea.attn_fwd(q, k, v, scale=inp.scale, causal=True)
        assert ea.attn_status() == ea.ATTN_ERR_TIMEOUT
        assert ea.attn_status() == ea.ATTN_OK  # reading clears it
    finally:
        ea.attn_debug_skip_load(-1)
        ea.attn_set_wait_limit_ms(prev_limit)
    o, lse = ea.attn_fwd(q, k, v, scale=inp.scale, causal=True)
    assert ea.attn_status() == ea.ATTN_OK
    ro, rl = oracle.fwd(inp.q, inp.k, inp.v, inp.scale, True)
    assert _within(o, ro, 1e-2, 1e-2)        # the forward parity tests' bands
    assert _within(lse, rl, 1e-3, 0.0)


@pytest.mark.parametrize("skip", [0, 2])
def test_backward_expired_wait_reports_timeout_and_context_survives(ea, skip):
    # Both backward kernels skip their query-side load number `skip`; every CTA stops
    # at the bounded wait, and the next call is correct.
    inp = make_dense(1, 2, 640, 64, seed=7100, with_grad=True)
    q, k, v, do = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.do.cuda()
    o, lse = ea.attn_fwd(q, k, v, scale=inp.scale, causal=True)
    assert ea.attn_status() == ea.ATTN_OK
    prev_limit = ea.attn_set_wait_limit_ms(200)
    ea.attn_debug_skip_load(skip)
    try:
        ea.attn_bwd(q, k, v, o, lse, do, scale=inp.scale, causal=True)
        assert ea.attn_status() == ea.ATTN_ERR_TIMEOUT
    finally:
        ea.attn_debug_skip_load(-1)
        ea.attn_set_wait_limit_ms(prev_limit)
    dq, dk, dv = ea.attn_bwd(q, k, v, o, lse, do, scale=inp.scale, causal=True)
    assert ea.attn_status() == ea.ATTN_OK
    rq, rk, rv = oracle.bwd(inp.q, inp.k, inp.v, inp.do, inp.scale, True)
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        assert _within(got, ref, 2e-2, 2e-2)

