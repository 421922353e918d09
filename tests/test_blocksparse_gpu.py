"""Block-sparse attention (codechina FlashAttention article, §7.1 variant algorithms,
Block-Sparse FlashAttention) through the C ABI, against the float64 oracle with the
same per-head tile mask: a left-out (query tile, key tile) pair behaves as masked
scores, a query row left with no key gets O = 0 and lse = -inf.

Tolerances as the dense tests: O |err| <= 1e-2 + 1e-2 |ref|, lse |err| <= 1e-3 (and
-inf exactly where the oracle has -inf), gradients |err| <= 2e-2 + 2e-2 |ref|.
"""
import numpy as np
import pytest
import torch

import oracle
from attn_inputs import make_dense, tile_mask

pytestmark = pytest.mark.gpu

O_ATOL, O_RTOL, LSE_ATOL = 1e-2, 1e-2, 1e-3
G_ATOL, G_RTOL = 2e-2, 2e-2


@pytest.fixture(scope="module")
def ea():
    from exact_attention_123_b200 import build
    build.build()
    import exact_attention_123_b200 as m
    assert torch.cuda.is_available()
    return m


def _close(got, ref, atol, rtol, what):
    g = got.detach().double().cpu().numpy() if isinstance(got, torch.Tensor) else got
    assert not np.any(np.isnan(g)), f"{what}: NaN"
    bad = np.abs(g - ref) > atol + rtol * np.abs(ref)
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} out of tolerance; max err {np.abs(g - ref).max()}"


def _lse(got, ref):
    g = got.detach().double().cpu().numpy()
    ninf = np.isneginf(ref)
    assert np.all(np.isneginf(g[ninf])), "rows with no key must have lse = -inf"
    assert np.all(np.isfinite(g[~ninf]))
    if (~ninf).any():
        assert np.abs(g[~ninf] - ref[~ninf]).max() <= LSE_ATOL


def _run(ea, inp, bm, causal):
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))
    bmd = bm.cuda()
    o = torch.full_like(q, float("nan"))
    lse = torch.full(q.shape[:3], float("nan"), device="cuda")
    ea.attn_fwd_blocksparse(q, k, v, bmd, o, lse, scale=inp.scale, causal=causal)
    dq, dk, dv = (torch.full_like(t, float("nan")) for t in (q, k, v))
    ea.attn_bwd_blocksparse(q, k, v, o, lse, do, bmd, dq, dk, dv, scale=inp.scale, causal=causal)
    assert ea.attn_status() == ea.ATTN_OK
    return o, lse, dq, dk, dv


CASES = [
    # B, H, N, d, causal, density, seed, emptied query-tile rows, emptied key-tile columns
    (2, 3, 700, 128, False, 0.5, 9001, [(0, 2)], [(1, 3)]),
    (2, 3, 700, 128, True, 0.6, 9002, [(2, 5)], [(0, 0)]),
    (1, 4, 1024, 64, False, 0.3, 9003, [(3, 7)], []),
    (1, 2, 640, 64, True, 0.5, 9004, [], [(1, 4)]),
]


@pytest.mark.parametrize("B,H,N,d,causal,density,seed,er,ec", CASES)
def test_blocksparse_matches_oracle(ea, B, H, N, d, causal, density, seed, er, ec):
    inp = make_dense(B, H, N, d, seed=seed, causal=causal, with_grad=True)
    bm = tile_mask(H, N, seed + 1, density, empty_rows=er, empty_cols=ec)
    o, lse, dq, dk, dv = _run(ea, inp, bm, causal)
    ro, rl = oracle.fwd(inp.q, inp.k, inp.v, inp.scale, causal, block_mask=bm.numpy())
    _close(o, ro, O_ATOL, O_RTOL, "O")
    _lse(lse, rl)
    gq, gk, gv = oracle.bwd(inp.q, inp.k, inp.v, inp.do, inp.scale, causal, block_mask=bm.numpy())
    _close(dq, gq, G_ATOL, G_RTOL, "dQ")
    _close(dk, gk, G_ATOL, G_RTOL, "dK")
    _close(dv, gv, G_ATOL, G_RTOL, "dV")
    # the emptied query tiles: O = 0 and lse = -inf exactly, dQ = 0
    for h, i in er:
        rows = slice(i * 128, min(N, (i + 1) * 128))
        assert torch.all(o[:, h, rows] == 0) and torch.all(torch.isneginf(lse[:, h, rows]))
        assert torch.all(dq[:, h, rows] == 0)
    # key tiles no query reaches: dK = dV = 0 exactly
    for h, j in ec:
        rows = slice(j * 128, min(N, (j + 1) * 128))
        assert torch.all(dk[:, h, rows] == 0) and torch.all(dv[:, h, rows] == 0)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_full_mask_is_the_dense_path(ea, d, causal):
    # every pair kept: the block-sparse kernels do the dense kernels' arithmetic, so
    # O and lse match bit for bit where both sweep the key tiles in the same order, and
    # dK, dV (from the same O and lse) bit for bit; dQ up to the order in which the key
    # tiles' fp32 contributions reach its accumulator (a few bf16 ulps at most).  The
    # one order difference: at d = 64 the dense causal forward sweeps the second query
    # tile of each 256-row unit (rows 128-255 of it) from its diagonal key tile, where
    # the running max moves at other tiles.  P is rounded to bf16 (relative error <= 2^-9)
    # on that running max's scale before P V, so those rows' O may differ by twice that
    # times sum_j P_j |v_j| / l <= max |v|, plus a bf16 rounding step of O; lse by at
    # most twice the relative error of the exponentials (at d = 64 one column pair in
    # eight comes from the FMA-pipe cubic, relative error <= 1.02e-4, whose arguments
    # shift with the running max), plus float rounding.
    N = 520
    inp = make_dense(2, 2, N, d, seed=9100 + d, causal=causal, with_grad=True)
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))
    bm = torch.ones((2, 5, 5), dtype=torch.uint8)
    o, lse, dq, dk, dv = _run(ea, inp, bm, causal)
    o2, lse2 = ea.attn_fwd(q, k, v, scale=inp.scale, causal=causal)
    dq2, dk2, dv2 = ea.attn_bwd(q, k, v, o, lse, do, scale=inp.scale, causal=causal)
    reordered = torch.zeros(N, dtype=torch.bool)
    if d == 64 and causal:
        for u0 in range(0, N, 256):
            reordered[u0 + 128:u0 + 256] = True
    same = ~reordered
    assert torch.equal(o[:, :, same], o2[:, :, same]) and torch.equal(lse[:, :, same], lse2[:, :, same])
    if reordered.any():
        a, b = o[:, :, reordered].double(), o2[:, :, reordered].double()
        vmax = inp.v.double().abs().max().item()
        assert torch.all((a - b).abs() <= 2 ** -7 * b.abs() + 2 ** -8 * vmax)
        assert torch.all((lse[:, :, reordered] - lse2[:, :, reordered]).abs() <= 2 * 1.02e-4 + 1e-5)
    assert torch.equal(dk, dk2) and torch.equal(dv, dv2)
    a, b = dq.double(), dq2.double()
    assert torch.all((a - b).abs() <= 2 ** -6 * b.abs() + 1e-3)


def test_empty_mask(ea):
    inp = make_dense(1, 2, 300, 128, seed=9200, causal=False, with_grad=True)
    bm = torch.zeros((2, 3, 3), dtype=torch.uint8)
    o, lse, dq, dk, dv = _run(ea, inp, bm, False)
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))
    for t in (dq, dk, dv):
        assert torch.all(t == 0)


def test_bench_size_sampled_slices(ea):
    # the bench's shape (B2 H16 N4096 d128, causal) with half the tile pairs left out;
    # two (b, h) slices checked against the oracle
    B, H, N, d = 2, 16, 4096, 128
    inp = make_dense(B, H, N, d, seed=9300, causal=True, with_grad=True)
    bm = tile_mask(H, N, 9301, 0.5, empty_rows=[(5, 17)], empty_cols=[(21 % H, 3)])
    o, lse, dq, dk, dv = _run(ea, inp, bm, True)
    slices = [0 * H + 5, 1 * H + 21 % H]
    ro, rl = oracle.fwd(inp.q, inp.k, inp.v, inp.scale, True, block_mask=bm.numpy(), slices=slices)
    gq, gk, gv = oracle.bwd(inp.q, inp.k, inp.v, inp.do, inp.scale, True, block_mask=bm.numpy(), slices=slices)
    for s in slices:
        b, h = divmod(s, H)
        _close(o[b, h], ro[b, h], O_ATOL, O_RTOL, f"O[{b},{h}]")
        _lse(lse[b, h], rl[b, h])
        _close(dq[b, h], gq[b, h], G_ATOL, G_RTOL, f"dQ[{b},{h}]")
        _close(dk[b, h], gk[b, h], G_ATOL, G_RTOL, f"dK[{b},{h}]")
        _close(dv[b, h], gv[b, h], G_ATOL, G_RTOL, f"dV[{b},{h}]")
