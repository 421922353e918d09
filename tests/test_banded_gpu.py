"""The banded unit order (and the claimed deal that goes with it) on small problems.

The single-pass backward walks its units in bands of (sequence, head) slices when
their Q, dO and dQ far exceed the L2 cache, and the packed and block-sparse forwards
do so for K and V; at test sizes that never happens, so attn_debug_force_band forces
bands of a few slices.  The results are checked against the float64 oracle (same
tolerances as the other parity tests) and against the same call without bands: a
unit's arithmetic does not depend on the order, so O, lse, dK and dV agree bit for
bit, dQ up to the order in which the key tiles' fp32 contributions reach its
accumulator.
"""
import numpy as np
import pytest
import torch

import oracle
from attn_inputs import make_dense, make_varlen, padding_key_mask, tile_mask

pytestmark = pytest.mark.gpu

O_ATOL, O_RTOL = 1e-2, 1e-2
LSE_ATOL = 1e-3
G_ATOL, G_RTOL = 2e-2, 2e-2


@pytest.fixture(scope="module")
def ea():
    from exact_attention_123_b200 import build
    build.build()
    import exact_attention_123_b200 as m
    return m


def _close(got, ref, atol, rtol, what):
    g = got.detach().cpu().double().numpy()
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    bad = np.abs(g - ref) > atol + rtol * np.abs(ref)
    assert not bad.any(), f"{what}: {bad.sum()}/{bad.size} out of tolerance"


def _lse(got, ref):
    g = got.detach().cpu().double().numpy()
    ninf = np.isneginf(ref)
    assert np.array_equal(np.isneginf(g), ninf)
    assert np.abs(g[~ninf] - ref[~ninf]).max() <= LSE_ATOL


def _dq_close(a, b):
    a, b = a.double(), b.double()
    assert torch.all((a - b).abs() <= 2 ** -6 * b.abs() + 1e-3)


def _banded(ea, slices, fn):
    prev = ea.attn_debug_force_band(slices)
    try:
        return fn()
    finally:
        ea.attn_debug_force_band(prev)


def test_force_band_setter_round_trip(ea):
    assert ea.attn_debug_force_band(3) == 0
    assert ea.attn_debug_force_band(0) == 3


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
def test_backward_in_bands_matches_oracle(ea, d, causal):
    inp = make_dense(2, 3, 300, d, seed=9300 + d, causal=causal, with_grad=True)  # 6 slices: bands of 4 and 2
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))
    o, lse = ea.attn_fwd(q, k, v, scale=inp.scale, causal=causal)

    def bwd():
        dq, dk, dv = (torch.full_like(t, float("nan")) for t in (q, k, v))
        ea.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, scale=inp.scale, causal=causal)
        assert ea.attn_status() == ea.ATTN_OK
        return dq, dk, dv

    dq, dk, dv = _banded(ea, 4, bwd)
    rq, rk, rv = oracle.bwd(inp.q, inp.k, inp.v, inp.do, inp.scale, causal)
    _close(dq, rq, G_ATOL, G_RTOL, "dQ")
    _close(dk, rk, G_ATOL, G_RTOL, "dK")
    _close(dv, rv, G_ATOL, G_RTOL, "dV")
    dq2, dk2, dv2 = bwd()  # the automatic (unbanded, dealt) order
    assert torch.equal(dk, dk2) and torch.equal(dv, dv2)
    _dq_close(dq, dq2)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
def test_packed_forward_and_backward_in_bands_match_oracle(ea, d, causal):
    lengths = [1, 130, 257, 64, 300, 128]  # 6 sequences x 3 heads = 18 slices: bands of 4 (last 2)
    inp = make_varlen(lengths, 3, d, seed=9400 + d, with_grad=True)
    keep = padding_key_mask(lengths, seed=9401, pad_frac=0.05, extra_frac=0.05)
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))
    cu, kk = inp.cu_seqlens.cuda(), keep.cuda()
    kw = dict(scale=inp.scale, causal=causal, cu_seqlens=cu, key_keep=kk, max_seqlen=max(lengths))

    def run():
        o, lse = ea.attn_fwd(q, k, v, **kw)
        dq, dk, dv = (torch.full_like(t, float("nan")) for t in (q, k, v))
        ea.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, **kw)
        assert ea.attn_status() == ea.ATTN_OK
        return o, lse, dq, dk, dv

    o, lse, dq, dk, dv = _banded(ea, 4, run)
    ro, rl = oracle.fwd(inp.q, inp.k, inp.v, inp.scale, causal, cu_seqlens=inp.cu_seqlens, key_keep=keep)
    _close(o, ro, O_ATOL, O_RTOL, "O")
    _lse(lse, rl)
    rq, rk, rv = oracle.bwd(inp.q, inp.k, inp.v, inp.do, inp.scale, causal, cu_seqlens=inp.cu_seqlens,
                            key_keep=keep)
    _close(dq, rq, G_ATOL, G_RTOL, "dQ")
    _close(dk, rk, G_ATOL, G_RTOL, "dK")
    _close(dv, rv, G_ATOL, G_RTOL, "dV")
    o2, lse2, dq2, dk2, dv2 = run()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    assert torch.equal(dk, dk2) and torch.equal(dv, dv2)
    _dq_close(dq, dq2)


@pytest.mark.parametrize("d", [64, 128])
def test_blocksparse_in_bands_matches_oracle(ea, d):
    B, H, N, causal = 2, 3, 700, True
    inp = make_dense(B, H, N, d, seed=9500 + d, causal=causal, with_grad=True)
    bm = tile_mask(H, N, 9501, 0.5)
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))
    bmd = bm.cuda()

    def run():
        o, lse = ea.attn_fwd_blocksparse(q, k, v, bmd, scale=inp.scale, causal=causal)
        dq, dk, dv = (torch.full_like(t, float("nan")) for t in (q, k, v))
        ea.attn_bwd_blocksparse(q, k, v, o, lse, do, bmd, dq, dk, dv, scale=inp.scale, causal=causal)
        assert ea.attn_status() == ea.ATTN_OK
        return o, lse, dq, dk, dv

    o, lse, dq, dk, dv = _banded(ea, 2, run)
    ro, rl = oracle.fwd(inp.q, inp.k, inp.v, inp.scale, causal, block_mask=bm.numpy())
    _close(o, ro, O_ATOL, O_RTOL, "O")
    _lse(lse, rl)
    gq, gk, gv = oracle.bwd(inp.q, inp.k, inp.v, inp.do, inp.scale, causal, block_mask=bm.numpy())
    _close(dq, gq, G_ATOL, G_RTOL, "dQ")
    _close(dk, gk, G_ATOL, G_RTOL, "dK")
    _close(dv, gv, G_ATOL, G_RTOL, "dV")
    o2, lse2, dq2, dk2, dv2 = run()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)
    assert torch.equal(dk, dk2) and torch.equal(dv, dv2)
    _dq_close(dq, dq2)
