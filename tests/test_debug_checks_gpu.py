"""The debug library (libattn_debug.so: the same kernels built with LIBATTN_DEBUG=1).

Its pipeline consistency checks (every bounded mbarrier wait finds the next phase of
its barrier still open; the forward's K/V ring fills carry {unit rank, key tile, fill
number} tags that the MMA issuer checks; at exit the forward's roles agree on the units,
fills and S phases they processed; the single-pass backward's Q stage fills carry {unit
rank, query tile, pair number} tags and its loader, issuer, math and drain warps agree
on their units and pairs) must pass on every entry point and leave the results
unchanged: each call is made with the release library and with the debug library on
the same inputs, and the outputs must agree bit for bit (dQ of the single-pass backward
up to the order in which the key tiles' fp32 contributions reach its accumulator, as in
the other tests).  A tag written wrong on purpose (attn_debug_corrupt_tag) must be
reported as ATTN_ERR_DEBUG_CHECK, after which a normal call runs clean.
"""
import pytest
import torch

from attn_inputs import make_dense, make_fp8, make_varlen, padding_key_mask, tile_mask

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ea():
    from exact_attention_123_b200 import build
    build.build()
    import exact_attention_123_b200 as m
    prev = m.use_debug_library(False)
    yield m
    m.use_debug_library(prev)


def both(ea, fn):
    """fn() with the release library, then with the debug library (status checked on each)."""
    out = []
    for debug in (False, True):
        ea.use_debug_library(debug)
        assert ea.attn_debug_checks() == debug
        res = fn()
        torch.cuda.synchronize()
        st = ea.attn_status()
        assert st == ea.ATTN_OK, f"debug={debug}: {ea.attn_strerror(st)}"
        out.append([t.clone() for t in res])
    ea.use_debug_library(False)
    return out


def same(a, b):
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def dq_close(a, b):
    a, b = a.double(), b.double()
    assert torch.all((a - b).abs() <= 2 ** -6 * b.abs() + 1e-3)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
def test_dense_forward_and_backwards(ea, d, causal):
    inp = make_dense(2, 3, 700, d, seed=9700 + d, causal=causal, with_grad=True)
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))

    def run():
        o, lse = ea.attn_fwd(q, k, v, scale=inp.scale, causal=causal)
        g = ea.attn_bwd(q, k, v, o, lse, do, scale=inp.scale, causal=causal)
        gd = ea.attn_bwd(q, k, v, o, lse, do, scale=inp.scale, causal=causal, deterministic=True)
        return (o, lse) + tuple(g) + tuple(gd)

    rel, dbg = both(ea, run)
    same(rel[:2], dbg[:2])            # O, lse
    dq_close(dbg[2], rel[2])          # single-pass dQ
    same(rel[3:5], dbg[3:5])          # dK, dV
    same(rel[5:], dbg[5:])            # the deterministic backward


@pytest.mark.parametrize("d", [64, 128])
def test_packed_masked_and_banded(ea, d):
    lengths = [1, 130, 257, 64, 300, 128]
    inp = make_varlen(lengths, 3, d, seed=9800 + d, with_grad=True)
    keep = padding_key_mask(lengths, seed=9801, pad_frac=0.05, extra_frac=0.05).cuda()
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))
    kw = dict(scale=inp.scale, causal=True, cu_seqlens=inp.cu_seqlens.cuda(), key_keep=keep, max_seqlen=max(lengths))

    def run():
        outs = []
        for band in (0, 4):  # automatic order, then forced bands of 4 slices (claimed units)
            prev = ea.attn_debug_force_band(band)
            try:
                o, lse = ea.attn_fwd(q, k, v, **kw)
                outs += [o, lse] + list(ea.attn_bwd(q, k, v, o, lse, do, **kw))
            finally:
                ea.attn_debug_force_band(prev)
        return outs

    rel, dbg = both(ea, run)
    for i in (0, 5):
        same(rel[i:i + 2], dbg[i:i + 2])
        dq_close(dbg[i + 2], rel[i + 2])
        same(rel[i + 3:i + 5], dbg[i + 3:i + 5])


@pytest.mark.parametrize("d", [64, 128])
def test_blocksparse(ea, d):
    inp = make_dense(2, 3, 700, d, seed=9900 + d, causal=True, with_grad=True)
    bm = tile_mask(3, 700, 9901, 0.5).cuda()
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))

    def run():
        o, lse = ea.attn_fwd_blocksparse(q, k, v, bm, scale=inp.scale, causal=True)
        dq, dk, dv = (torch.empty_like(t) for t in (q, k, v))
        ea.attn_bwd_blocksparse(q, k, v, o, lse, do, bm, dq, dk, dv, scale=inp.scale, causal=True)
        return o, lse, dq, dk, dv

    rel, dbg = both(ea, run)
    same(rel[:2], dbg[:2])
    dq_close(dbg[2], rel[2])
    same(rel[3:], dbg[3:])


@pytest.mark.parametrize("d", [64, 128])
def test_fp8_forward(ea, d):
    inp = make_fp8(2, 3, 700, d, seed=9950 + d, causal=True)
    q8, k8, v8 = inp.q8.cuda(), inp.k8.cuda(), inp.v8.cuda()

    def run():
        return ea.attn_fwd_fp8(q8, k8, v8, inp.q_scale, inp.k_scale, inp.v_scale, scale=inp.scale, causal=True)

    rel, dbg = both(ea, run)
    same(rel, dbg)


@pytest.mark.parametrize("d", [64, 128])
def test_fp8_blocksparse_forward(ea, d):
    inp = make_fp8(2, 3, 700, d, seed=9960 + d, causal=True)
    q8, k8, v8 = inp.q8.cuda(), inp.k8.cuda(), inp.v8.cuda()
    bm = tile_mask(3, 700, 9961, 0.5, empty_rows=[(1, 2)]).cuda()

    def run():
        return ea.attn_fwd_fp8_blocksparse(q8, k8, v8, inp.q_scale, inp.k_scale, inp.v_scale, bm, scale=inp.scale,
                                           causal=True)

    rel, dbg = both(ea, run)
    same(rel, dbg)


def test_corrupted_ring_tag_is_reported_then_clean(ea):
    inp = make_dense(1, 2, 1024, 128, seed=9990, causal=False)
    q, k, v = (t.cuda() for t in (inp.q, inp.k, inp.v))
    ref = ea.attn_fwd(q, k, v, scale=inp.scale, causal=False)
    assert ea.attn_status() == ea.ATTN_OK
    # the release library writes no tags: there the hook changes nothing
    ea.attn_debug_corrupt_tag(3)
    try:
        same(ref, ea.attn_fwd(q, k, v, scale=inp.scale, causal=False))
        assert ea.attn_status() == ea.ATTN_OK
    finally:
        ea.attn_debug_corrupt_tag(-1)
    ea.use_debug_library(True)  # (each library keeps its own hooks and status word)
    try:
        ea.attn_debug_corrupt_tag(3)
        try:
            ea.attn_fwd(q, k, v, scale=inp.scale, causal=False)
            assert ea.attn_status() == ea.ATTN_ERR_DEBUG_CHECK
        finally:
            ea.attn_debug_corrupt_tag(-1)
        same(ref, ea.attn_fwd(q, k, v, scale=inp.scale, causal=False))
        assert ea.attn_status() == ea.ATTN_OK
    finally:
        ea.use_debug_library(False)


def test_corrupted_backward_tag_is_reported_then_clean(ea):
    inp = make_dense(1, 2, 1024, 128, seed=9991, causal=True, with_grad=True)
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))
    o, lse = ea.attn_fwd(q, k, v, scale=inp.scale, causal=True)
    ref = ea.attn_bwd(q, k, v, o, lse, do, scale=inp.scale, causal=True)
    assert ea.attn_status() == ea.ATTN_OK
    ea.use_debug_library(True)
    try:
        ea.attn_debug_corrupt_tag(2)  # the third tile pair of every CTA
        try:
            ea.attn_bwd(q, k, v, o, lse, do, scale=inp.scale, causal=True)
            assert ea.attn_status() == ea.ATTN_ERR_DEBUG_CHECK
        finally:
            ea.attn_debug_corrupt_tag(-1)
        got = ea.attn_bwd(q, k, v, o, lse, do, scale=inp.scale, causal=True)
        assert ea.attn_status() == ea.ATTN_OK
        dq_close(got[0], ref[0])
        same(got[1:], ref[1:])
    finally:
        ea.use_debug_library(False)


def test_bench_shape_under_checks(ea):
    # the bench workload at full size (512 forward units and 1024 backward units on 148
    # CTAs): no check fires and the results equal the release library's
    inp = make_dense(2, 16, 4096, 128, seed=5, causal=True, with_grad=True)
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))

    def run():
        o, lse = ea.attn_fwd(q, k, v, scale=inp.scale, causal=True)
        return (o, lse) + tuple(ea.attn_bwd(q, k, v, o, lse, do, scale=inp.scale, causal=True))

    rel, dbg = both(ea, run)
    same(rel[:2], dbg[:2])
    dq_close(dbg[2], rel[2])
    same(rel[3:], dbg[3:])


def test_packed_workload_under_checks(ea):
    # 8 packed sequences of U[256, 4096] tokens, 32 heads, d = 128, key padding: large enough
    # that the forward and the single-pass backward walk their claimed units in L2-sized bands
    # of slices on their own
    from attn_inputs import draw_lengths
    lengths = draw_lengths(8, 256, 4096, 40)
    keep = padding_key_mask(lengths, 41).cuda()
    inp = make_varlen(lengths, 32, 128, 4, True, keep.cpu(), with_grad=True)
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))
    kw = dict(scale=inp.scale, causal=True, cu_seqlens=inp.cu_seqlens.cuda(), key_keep=keep, max_seqlen=max(lengths))

    def run():
        o, lse = ea.attn_fwd(q, k, v, **kw)
        return (o, lse) + tuple(ea.attn_bwd(q, k, v, o, lse, do, **kw))

    rel, dbg = both(ea, run)
    same(rel[:2], dbg[:2])
    dq_close(dbg[2], rel[2])
    same(rel[3:], dbg[3:])
