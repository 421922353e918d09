"""Seeded random configurations through the C ABI against the float64 oracle.

The other parity files pick their shapes by hand (tile edges, empty rows, the
workloads' sizes).  Here a seeded generator draws whole configurations -- the
layout (dense, dense with a key mask, packed sequences with a key mask, tile mask,
e4m3, e4m3 with a tile mask), d, causal, batch, heads, lengths, mask densities --
so that combinations nobody listed are run too.  Every case runs the forward and,
for the bf16 layouts, both backward algorithms, and compares each output element
with the oracle at the tolerances of the hand-picked tests: O |err| <= 1e-2 +
1e-2 |ref|, lse |err| <= 1e-3 (and -inf exactly where the oracle's is), gradients
|err| <= 2e-2 + 2e-2 |ref|; the e4m3 outputs against the bound derived in
test_fp8_gpu.py.
"""
import numpy as np
import pytest
import torch

import oracle
import test_fp8_gpu as f8
from attn_inputs import make_dense, make_fp8, make_varlen, padding_key_mask, tile_mask

pytestmark = pytest.mark.gpu

O_ATOL, O_RTOL, LSE_ATOL = 1e-2, 1e-2, 1e-3
G_ATOL, G_RTOL = 2e-2, 2e-2
KINDS = ("dense", "dense_keymask", "varlen", "blocksparse", "fp8", "fp8_blocksparse")
N_CASES = 72


def draw(case: int) -> dict:
    """Configuration `case` (0 .. N_CASES-1): every 24 consecutive cases take every
    (layout, d, causal) combination once; the rest is drawn from a generator seeded
    by the case number."""
    g = np.random.default_rng(20_000 + case)
    c = {"kind": KINDS[case % len(KINDS)], "d": (64, 128)[(case // len(KINDS)) % 2],
         "causal": bool((case // (2 * len(KINDS))) % 2), "seed": 20_000 + 100 * case}
    # lengths: mostly anywhere in [1, 900], sometimes on or next to a tile edge
    edge = [1, 127, 128, 129, 255, 256, 257, 384, 640]
    pick = lambda: int(g.choice(edge)) if g.random() < 0.3 else int(g.integers(1, 901))
    if c["kind"] == "varlen":
        c["lengths"] = [pick() for _ in range(int(g.integers(1, 7)))]
        c["H"] = int(g.integers(1, 4))
    else:
        c.update(B=int(g.integers(1, 4)), H=int(g.integers(1, 5)), N=pick())
    if c["kind"] in ("blocksparse", "fp8_blocksparse"):
        c["density"] = float(g.choice([0.15, 0.5, 0.85]))
    if c["kind"] == "dense_keymask":
        c["keep_frac"] = float(g.choice([0.3, 0.8, 0.97]))
    return c


def _np(t):
    return t.detach().cpu().to(torch.float64).numpy()


def close(got, ref, atol, rtol, what):
    g = _np(got)
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    bad = np.abs(g - ref) > atol + rtol * np.abs(ref)
    assert not bad.any(), f"{what}: {bad.sum()}/{bad.size} out of tolerance; max err {np.abs(g - ref).max():.3g}"


def lse_close(got, ref):
    g = _np(got)
    ninf = np.isneginf(ref)
    assert np.all(np.isneginf(g[ninf])), "rows with no visible key must have lse = -inf"
    assert np.all(np.isfinite(g[~ninf]))
    if (~ninf).any():
        assert np.abs(g[~ninf] - ref[~ninf]).max() <= LSE_ATOL


@pytest.fixture(scope="module")
def ea():
    from exact_attention_123_b200 import build
    build.build()
    import exact_attention_123_b200 as m
    return m


def test_the_draws_cover_every_combination():
    combos = {(k, d, cz) for k in KINDS for d in (64, 128) for cz in (True, False)}
    for start in range(0, N_CASES, 24):
        cs = [draw(i) for i in range(start, start + 24)]
        assert {(c["kind"], c["d"], c["causal"]) for c in cs} == combos


@pytest.mark.parametrize("case", range(N_CASES))
def test_random_config(ea, case):
    c = draw(case)
    kind, d, causal = c["kind"], c["d"], c["causal"]
    if kind.startswith("fp8"):
        inp = make_fp8(c["B"], c["H"], c["N"], d, seed=c["seed"], causal=causal)
        q8, k8, v8 = inp.q8.cuda(), inp.k8.cuda(), inp.v8.cuda()
        o = torch.full(q8.shape, float("nan"), device="cuda", dtype=torch.bfloat16)
        lse = torch.full(q8.shape[:3], float("nan"), device="cuda")
        bm = None
        if kind == "fp8_blocksparse":
            bm = tile_mask(c["H"], c["N"], c["seed"] + 1, c["density"])
            ea.attn_fwd_fp8_blocksparse(q8, k8, v8, inp.q_scale, inp.k_scale, inp.v_scale, bm.cuda(), o, lse,
                                        scale=inp.scale, causal=causal)
        else:
            ea.attn_fwd_fp8(q8, k8, v8, inp.q_scale, inp.k_scale, inp.v_scale, o, lse, scale=inp.scale,
                            causal=causal)
        assert ea.attn_status() == ea.ATTN_OK
        f8.check(inp, _np(o), _np(lse), causal, block_mask=bm)
        return

    keep = bm = cu = None
    if kind == "varlen":
        inp = make_varlen(c["lengths"], c["H"], d, seed=c["seed"], causal=causal, with_grad=True)
        keep = padding_key_mask(c["lengths"], seed=c["seed"] + 1, pad_frac=0.05, extra_frac=0.05)
        cu = inp.cu_seqlens
    else:
        inp = make_dense(c["B"], c["H"], c["N"], d, seed=c["seed"], causal=causal, with_grad=True)
        if kind == "dense_keymask":
            gk = torch.Generator("cpu").manual_seed(c["seed"] + 1)
            keep = (torch.rand(c["B"], c["N"], generator=gk) < c["keep_frac"]).to(torch.uint8)
        if kind == "blocksparse":
            bm = tile_mask(c["H"], c["N"], c["seed"] + 1, c["density"])
    q, k, v, do = (t.cuda() for t in (inp.q, inp.k, inp.v, inp.do))
    kw = dict(scale=inp.scale, causal=causal)
    if bm is not None:
        o, lse = ea.attn_fwd_blocksparse(q, k, v, bm.cuda(), **kw)
    else:
        kw.update(key_keep=None if keep is None else keep.cuda(), cu_seqlens=None if cu is None else cu.cuda(),
                  max_seqlen=inp.N if cu is not None else None)
        o, lse = ea.attn_fwd(q, k, v, **kw)
    assert ea.attn_status() == ea.ATTN_OK
    okw = dict(cu_seqlens=cu, key_keep=keep, block_mask=None if bm is None else bm.numpy())
    ro, rl = oracle.fwd(inp.q, inp.k, inp.v, inp.scale, causal, **okw)
    close(o, ro, O_ATOL, O_RTOL, "O")
    lse_close(lse, rl)
    rq, rk, rv = oracle.bwd(inp.q, inp.k, inp.v, inp.do, inp.scale, causal, **okw)
    for det in ((False,) if bm is not None else (False, True)):
        dq, dk, dv = (torch.full_like(t, float("nan")) for t in (q, k, v))
        if bm is not None:
            ea.attn_bwd_blocksparse(q, k, v, o, lse, do, bm.cuda(), dq, dk, dv, **kw)
        else:
            ea.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, deterministic=det, **kw)
        assert ea.attn_status() == ea.ATTN_OK
        tag = "deterministic" if det else "single pass"
        close(dq, rq, G_ATOL, G_RTOL, f"dQ ({tag})")
        close(dk, rk, G_ATOL, G_RTOL, f"dK ({tag})")
        close(dv, rv, G_ATOL, G_RTOL, f"dV ({tag})")
