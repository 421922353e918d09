"""Pins of the float64 CPU oracle against things other than itself.

Each test targets a plausible mistake: a dropped scale, a wrong mask index or
polarity, a missing max-subtraction, a transposed operand in the backward, an
off-by-one in the packed (varlen) slicing, or NaN on an empty row.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from attn_inputs import make_dense, make_varlen, padding_key_mask

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- helpers

def _num(s):
    s = s.strip()
    if s == "-inf":
        return -math.inf
    if s.startswith("ln"):
        return math.log(float(s[2:]))
    if "*ln" in s:
        a, b = s.split("*ln")
        return float(Fraction(a)) * math.log(float(b))
    return float(Fraction(s))


def brute_fwd(q, k, v, scale, causal, keep=None, allow=None):
    """Triple-loop forward on one head (lists of lists), naive exp(s)/sum exp(s).
    allow(i, j), if given, is an extra pair predicate (a tile mask)."""
    n, d = len(q), len(q[0])
    o = [[0.0] * d for _ in range(n)]
    lse = [0.0] * n
    for i in range(n):
        vis = [j for j in range(n) if (not causal or j <= i) and (keep is None or keep[j])
               and (allow is None or allow(i, j))]
        if not vis:
            lse[i] = -math.inf
            continue
        s = {j: scale * sum(q[i][c] * k[j][c] for c in range(d)) for j in vis}
        den = sum(math.exp(s[j]) for j in vis)
        for j in vis:
            p = math.exp(s[j]) / den
            for c in range(d):
                o[i][c] += p * v[j][c]
        lse[i] = math.log(den)
    return o, lse


def brute_bwd(q, k, v, do, scale, causal, keep=None, allow=None):
    """Backward by the chain rule through each row's softmax, written with loops."""
    n, d = len(q), len(q[0])
    dq = [[0.0] * d for _ in range(n)]
    dk = [[0.0] * d for _ in range(n)]
    dv = [[0.0] * d for _ in range(n)]
    for i in range(n):
        vis = [j for j in range(n) if (not causal or j <= i) and (keep is None or keep[j])
               and (allow is None or allow(i, j))]
        if not vis:
            continue
        s = {j: scale * sum(q[i][c] * k[j][c] for c in range(d)) for j in vis}
        den = sum(math.exp(s[j]) for j in vis)
        p = {j: math.exp(s[j]) / den for j in vis}
        # dL/dp_j = do_i . v_j ; softmax Jacobian dp_j/ds_t = p_j (delta_jt - p_t)
        g = {j: sum(do[i][c] * v[j][c] for c in range(d)) for j in vis}
        for t in vis:
            ds = sum(g[j] * p[j] * ((1.0 if j == t else 0.0) - p[t]) for j in vis)
            for c in range(d):
                dq[i][c] += ds * scale * k[t][c]
                dk[t][c] += ds * scale * q[i][c]
        for j in vis:
            for c in range(d):
                dv[j][c] += p[j] * do[i][c]
    return dq, dk, dv


def rnd(shape, seed, sigma=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * sigma


# ---------------------------------------------------------------- golden (hand-derived)

def test_hand_example_forward():
    g = json.load(open(os.path.join(GOLDEN, "hand_example.json")))["forward"]
    q = np.array(g["q"]).reshape(1, 1, 3, 1)
    k = np.array([_num(x) for x in g["k_exact"]]).reshape(1, 1, 3, 1)
    v = np.array(g["v"]).reshape(1, 1, 3, 1)
    for case in g["cases"]:
        keep = np.array([case["key_keep"]], dtype=np.uint8)
        o, lse = oracle.fwd(q, k, v, 1.0, case["causal"], key_keep=keep)
        want_o = [_num(x) for x in case["o"]]
        want_l = [_num(x) for x in case["lse"]]
        np.testing.assert_allclose(o.reshape(-1), want_o, rtol=0, atol=1e-12, err_msg=case["name"])
        for got, want in zip(lse.reshape(-1), want_l):
            if want == -math.inf:
                assert got == -math.inf, case["name"]
            else:
                assert abs(got - want) < 1e-12, case["name"]


def test_hand_example_backward():
    g = json.load(open(os.path.join(GOLDEN, "hand_example.json")))["backward"]
    sh = (1, 1, 2, 1)
    q = np.array(g["q"]).reshape(sh)
    k = np.array([_num(x) for x in g["k_exact"]]).reshape(sh)
    v = np.array(g["v"]).reshape(sh)
    do = np.array(g["do"]).reshape(sh)
    dq, dk, dv = oracle.bwd(q, k, v, do, 1.0, False)
    np.testing.assert_allclose(dq.reshape(-1), [_num(x) for x in g["dq"]], atol=1e-12)
    np.testing.assert_allclose(dk.reshape(-1), [_num(x) for x in g["dk"]], atol=1e-12)
    np.testing.assert_allclose(dv.reshape(-1), [_num(x) for x in g["dv"]], atol=1e-12)


# ---------------------------------------------------------------- T1 brute force

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("masked", [False, True])
def test_brute_force_forward_backward(causal, masked):
    B, H, N, d = 1, 2, 11, 5
    q, k, v, do = (rnd((B, H, N, d), s) for s in (1, 2, 3, 4))
    keep = None
    if masked:
        keep = np.ones((B, N), np.uint8)
        keep[0, [0, 3, 7]] = 0      # row 0 is fully masked when causal
    scale = 0.37
    o, lse = oracle.fwd(q, k, v, scale, causal, key_keep=keep)
    dq, dk, dv = oracle.bwd(q, k, v, do, scale, causal, key_keep=keep)
    for h in range(H):
        kk = None if keep is None else list(keep[0])
        bo, bl = brute_fwd(q[0, h].tolist(), k[0, h].tolist(), v[0, h].tolist(), scale, causal, kk)
        np.testing.assert_allclose(o[0, h], bo, rtol=0, atol=1e-12)
        for got, want in zip(lse[0, h], bl):
            assert (got == want == -math.inf) or abs(got - want) < 1e-12
        gq, gk, gv = brute_bwd(q[0, h].tolist(), k[0, h].tolist(), v[0, h].tolist(),
                               do[0, h].tolist(), scale, causal, kk)
        np.testing.assert_allclose(dq[0, h], gq, rtol=0, atol=1e-12)
        np.testing.assert_allclose(dk[0, h], gk, rtol=0, atol=1e-12)
        np.testing.assert_allclose(dv[0, h], gv, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- T2 finite differences

@pytest.mark.parametrize("causal", [False, True])
def test_finite_differences(causal):
    B, H, N, d = 1, 1, 9, 4
    q, k, v, G = (rnd((B, H, N, d), s) for s in (11, 12, 13, 14))
    keep = np.ones((B, N), np.uint8)
    keep[0, 0] = 0   # causal: row 0 fully masked
    keep[0, 5] = 0
    scale = 0.61

    def loss(qq, kk, vv):
        o, _ = oracle.fwd(qq, kk, vv, scale, causal, key_keep=keep)
        return float(np.sum(o * G))

    dq, dk, dv = oracle.bwd(q, k, v, G, scale, causal, key_keep=keep)
    h = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        err = np.max(np.abs(num - grad)) / max(1e-12, np.max(np.abs(grad)))
        assert err < 1e-6, (name, err)
    # the masked key and (causal) the fully masked row carry exactly zero gradient
    assert np.all(dk[0, 0, 0] == 0) and np.all(dv[0, 0, 0] == 0)
    if causal:
        assert np.all(dq[0, 0, 0] == 0)


# ---------------------------------------------------------------- T3 rows of P sum to 1

@pytest.mark.parametrize("causal", [False, True])
def test_rows_of_p_sum_to_one(causal):
    # With V = identity, O_i is row i of P itself.
    N = 16
    q = rnd((1, 1, N, N), 21)
    k = rnd((1, 1, N, N), 22)
    v = np.eye(N).reshape(1, 1, N, N)
    keep = np.ones((1, N), np.uint8)
    keep[0, 0] = 0
    o, _ = oracle.fwd(q, k, v, 0.25, causal, key_keep=keep)
    P = o[0, 0]
    sums = P.sum(axis=1)
    for i in range(N):
        if causal and i == 0:
            assert sums[i] == 0.0
        else:
            assert abs(sums[i] - 1.0) < 1e-12
    assert np.all(P[:, 0] == 0.0)                     # masked key gets no weight
    if causal:
        assert np.all(np.triu(P, 1) == 0.0)           # nothing above the diagonal
    assert np.all(P >= 0.0)


# ---------------------------------------------------------------- T4 constant V

def test_constant_v_rows():
    N, d = 13, 6
    q, k = rnd((1, 2, N, d), 31), rnd((1, 2, N, d), 32)
    c = rnd((d,), 33)
    v = np.broadcast_to(c, (1, 2, N, d)).copy()
    for causal in (False, True):
        o, _ = oracle.fwd(q, k, v, 0.5, causal)
        np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), atol=1e-12)


# ---------------------------------------------------------------- T5 causal first row

def test_causal_first_row():
    N, d = 10, 7
    q, k, v = rnd((2, 3, N, d), 41), rnd((2, 3, N, d), 42), rnd((2, 3, N, d), 43)
    scale = 0.3
    o, lse = oracle.fwd(q, k, v, scale, True)
    np.testing.assert_array_equal(o[:, :, 0], v[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], scale * np.sum(q[:, :, 0] * k[:, :, 0], -1), atol=1e-13)


# ---------------------------------------------------------------- T6 online-softmax equivalence

def test_zero_q_prefix_mean():
    N, d = 12, 5
    q = np.zeros((1, 1, N, d))
    k, v = rnd((1, 1, N, d), 51), rnd((1, 1, N, d), 52)
    o, lse = oracle.fwd(q, k, v, 0.9, True)
    for i in range(N):
        np.testing.assert_allclose(o[0, 0, i], v[0, 0, : i + 1].mean(0), atol=1e-13)
        assert abs(lse[0, 0, i] - math.log(i + 1)) < 1e-13
    o, lse = oracle.fwd(q, k, v, 0.9, False)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(v[0, 0].mean(0), (N, d)), atol=1e-13)
    np.testing.assert_allclose(lse[0, 0], math.log(N), atol=1e-13)


def online_softmax_tiled(q, k, v, scale, causal, tile):
    """The running-max / running-sum recurrence over key tiles, restated in float64
    ('4.5 注意力优化实战' 第三步 §1; codechina FlashAttention article §3.2)."""
    n, d = q.shape
    O = np.zeros((n, d))
    lse = np.zeros(n)
    for i in range(n):
        m_prev, l_prev, o = -math.inf, 0.0, np.zeros(d)
        for j0 in range(0, n, tile):
            js = [j for j in range(j0, min(n, j0 + tile)) if not causal or j <= i]
            if not js:
                continue
            s = np.array([scale * float(q[i] @ k[j]) for j in js])
            m_cur = max(m_prev, float(s.max()))
            corr = math.exp(m_prev - m_cur) if m_prev != -math.inf else 0.0
            p = np.exp(s - m_cur)
            l_prev = l_prev * corr + float(p.sum())
            o = o * corr + p @ v[js]
            m_prev = m_cur
        O[i] = o / l_prev
        lse[i] = m_prev + math.log(l_prev)
    return O, lse


@pytest.mark.parametrize("tile", [1, 7, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_tiled_recurrence_matches(tile, causal):
    N, d = 40, 8
    q, k, v = rnd((N, d), 61, 3.0), rnd((N, d), 62, 3.0), rnd((N, d), 63)
    o, lse = oracle.fwd(q[None, None], k[None, None], v[None, None], 0.4, causal)
    to, tl = online_softmax_tiled(q, k, v, 0.4, causal, tile)
    np.testing.assert_allclose(o[0, 0], to, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], tl, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- T7 mask semantics (packed)

def test_fully_masked_rows_are_zero_not_nan():
    lengths = [5, 9, 3]
    H, d = 2, 4
    inp = make_varlen(lengths, H, d, seed=71)
    keep = padding_key_mask(lengths, seed=72, pad_frac=0.34, extra_frac=0.0)
    o, lse = oracle.fwd(inp.q, inp.k, inp.v, 0.5, True, cu_seqlens=inp.cu_seqlens, key_keep=keep)
    assert not np.any(np.isnan(o))
    cu = inp.cu_seqlens.tolist()
    for b, n in enumerate(lengths):
        p = math.ceil(0.34 * n)
        for i in range(n):
            t = cu[b] + i
            if i < p:
                assert np.all(o[t] == 0.0) and np.all(lse[t] == -math.inf)
            else:
                assert np.all(np.isfinite(lse[t]))


def test_packed_layout_matches_per_sequence_dense():
    lengths = [7, 1, 12, 4]
    H, d = 3, 5
    inp = make_varlen(lengths, H, d, seed=81, with_grad=True)
    keep = torch.ones(sum(lengths), dtype=torch.uint8)
    keep[[2, 9, 20]] = 0
    o, lse = oracle.fwd(inp.q, inp.k, inp.v, 0.3, True, cu_seqlens=inp.cu_seqlens, key_keep=keep)
    dq, dk, dv = oracle.bwd(inp.q, inp.k, inp.v, inp.do, 0.3, True, cu_seqlens=inp.cu_seqlens, key_keep=keep)
    cu = inp.cu_seqlens.tolist()
    for b, n in enumerate(lengths):
        sl = slice(cu[b], cu[b + 1])
        to_dense = lambda x: x[sl].to(torch.float64).permute(1, 0, 2).unsqueeze(0).numpy()
        kk = keep[sl].numpy()[None]
        od, ld = oracle.fwd(to_dense(inp.q), to_dense(inp.k), to_dense(inp.v), 0.3, True, key_keep=kk)
        np.testing.assert_array_equal(o[sl], od[0].transpose(1, 0, 2))
        np.testing.assert_array_equal(lse[sl], ld[0].T)
        gq, gk, gv = oracle.bwd(to_dense(inp.q), to_dense(inp.k), to_dense(inp.v), to_dense(inp.do),
                                0.3, True, key_keep=kk)
        np.testing.assert_array_equal(dq[sl], gq[0].transpose(1, 0, 2))
        np.testing.assert_array_equal(dk[sl], gk[0].transpose(1, 0, 2))
        np.testing.assert_array_equal(dv[sl], gv[0].transpose(1, 0, 2))


# ---------------------------------------------------------------- T8 shift / permutation invariance

def test_key_shift_and_permutation_invariance():
    N, d = 14, 6
    q, k, v = rnd((1, 1, N, d), 91), rnd((1, 1, N, d), 92), rnd((1, 1, N, d), 93)
    u = rnd((d,), 94)
    scale = 0.45
    for causal in (False, True):
        o, lse = oracle.fwd(q, k, v, scale, causal)
        o2, lse2 = oracle.fwd(q, k + u, v, scale, causal)
        np.testing.assert_allclose(o2, o, atol=1e-12)
        np.testing.assert_allclose(lse2[0, 0], lse[0, 0] + scale * (q[0, 0] @ u), atol=1e-12)
    perm = np.random.default_rng(95).permutation(N)
    o, lse = oracle.fwd(q, k, v, scale, False)
    o3, lse3 = oracle.fwd(q, k[:, :, perm], v[:, :, perm], scale, False)
    np.testing.assert_allclose(o3, o, atol=1e-12)
    np.testing.assert_allclose(lse3, lse, atol=1e-12)


# ---------------------------------------------------------------- T9 backward identities

@pytest.mark.parametrize("causal", [False, True])
def test_backward_identities(causal):
    N, d = 17, 6
    q, k, v, do = (rnd((1, 2, N, d), s) for s in (101, 102, 103, 104))
    keep = np.ones((1, N), np.uint8)
    keep[0, [0, 1]] = 0          # causal: rows 0 and 1 fully masked
    dq, dk, dv = oracle.bwd(q, k, v, do, 0.35, causal, key_keep=keep)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    visible = np.ones(N, bool)
    if causal:
        visible[:2] = False
    np.testing.assert_allclose(dv.sum(axis=2), do[:, :, visible].sum(axis=2), atol=1e-12)


# ---------------------------------------------------------------- T10 library cross-check

def test_torch_float64_composition():
    inp = make_dense(2, 3, 33, 16, seed=111, with_grad=True)
    q, k, v, do = (t.to(torch.float64).requires_grad_(True) for t in (inp.q, inp.k, inp.v, inp.do))
    s = (q @ k.transpose(-1, -2)) * inp.scale
    s = s.masked_fill(torch.ones(33, 33, dtype=torch.bool).triu(1), float("-inf"))
    o = torch.softmax(s, -1) @ v
    lse = torch.logsumexp(s, -1)
    o.backward(do)
    oo, ll = oracle.fwd(inp.q, inp.k, inp.v, inp.scale, True)
    gq, gk, gv = oracle.bwd(inp.q, inp.k, inp.v, inp.do, inp.scale, True)
    np.testing.assert_allclose(oo, o.detach().numpy(), atol=1e-12)
    np.testing.assert_allclose(ll, lse.detach().numpy(), atol=1e-12)
    np.testing.assert_allclose(gq, q.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(gk, k.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(gv, v.grad.numpy(), atol=1e-11)


def test_slice_selection_leaves_others_untouched():
    inp = make_dense(2, 2, 9, 4, seed=121)
    o, lse = oracle.fwd(inp.q, inp.k, inp.v, 0.5, True, slices=[3])
    assert np.all(np.isnan(o[0])) and np.all(np.isnan(o[1, 0]))
    full, _ = oracle.fwd(inp.q, inp.k, inp.v, 0.5, True)
    np.testing.assert_array_equal(o[1, 1], full[1, 1])


# ---------------------------------------------------------------- block-sparse tile mask
# codechina FlashAttention article, §7.1 (Block-Sparse FlashAttention):
# a (query tile, key tile) pair either takes part as a whole or is left out.

def _tile_mask(H, nb, seed, density=0.6):
    return (np.random.default_rng(seed).random((H, nb, nb)) < density).astype(np.uint8)


@pytest.mark.parametrize("causal", [False, True])
def test_block_mask_brute_force(causal):
    B, H, N, d, blk = 1, 2, 11, 5, 3          # 4 x 4 tiles, the last one ragged
    q, k, v, do = (rnd((B, H, N, d), s) for s in (41, 42, 43, 44))
    nb = -(-N // blk)
    bm = _tile_mask(H, nb, 45)
    bm[0, 1, :] = 0                           # head 0: query rows 3-5 see no key at all
    scale = 0.53
    o, lse = oracle.fwd(q, k, v, scale, causal, block_mask=bm, block=blk)
    dq, dk, dv = oracle.bwd(q, k, v, do, scale, causal, block_mask=bm, block=blk)
    for h in range(H):
        allow = lambda i, j, h=h: bool(bm[h, i // blk, j // blk])
        bo, bl = brute_fwd(q[0, h].tolist(), k[0, h].tolist(), v[0, h].tolist(), scale, causal, None, allow)
        np.testing.assert_allclose(o[0, h], bo, rtol=0, atol=1e-12)
        for got, want in zip(lse[0, h], bl):
            assert (got == want == -math.inf) or abs(got - want) < 1e-12
        gq, gk, gv = brute_bwd(q[0, h].tolist(), k[0, h].tolist(), v[0, h].tolist(), do[0, h].tolist(),
                               scale, causal, None, allow)
        np.testing.assert_allclose(dq[0, h], gq, rtol=0, atol=1e-12)
        np.testing.assert_allclose(dk[0, h], gk, rtol=0, atol=1e-12)
        np.testing.assert_allclose(dv[0, h], gv, rtol=0, atol=1e-12)
    # the emptied query tile: O = 0, lse = -inf, no gradient flows through it
    assert np.all(o[0, 0, 3:6] == 0) and np.all(lse[0, 0, 3:6] == -math.inf)
    assert np.all(dq[0, 0, 3:6] == 0)


@pytest.mark.parametrize("causal", [False, True])
def test_block_mask_of_key_columns_equals_key_keep(causal):
    # leaving out key tile 2 for every query tile is the per-key mask of its keys
    B, H, N, d, blk = 2, 3, 20, 4, 4
    q, k, v, do = (rnd((B, H, N, d), s) for s in (51, 52, 53, 54))
    nb = N // blk
    bm = np.ones((H, nb, nb), np.uint8)
    bm[:, :, 2] = 0
    keep = np.ones((B, N), np.uint8)
    keep[:, 8:12] = 0
    a = oracle.fwd(q, k, v, 0.4, causal, block_mask=bm, block=blk)
    b = oracle.fwd(q, k, v, 0.4, causal, key_keep=keep)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    ga = oracle.bwd(q, k, v, do, 0.4, causal, block_mask=bm, block=blk)
    gb = oracle.bwd(q, k, v, do, 0.4, causal, key_keep=keep)
    for x, y in zip(ga, gb):
        np.testing.assert_array_equal(x, y)


def test_block_mask_single_tile_is_attention_on_that_tile():
    # query tile i with only key tile j left in is plain attention of those rows on
    # those keys (computed without any mask, on the cut-out tiles)
    B, H, N, d, blk = 1, 2, 12, 3, 4
    q, k, v = (rnd((B, H, N, d), s) for s in (61, 62, 63))
    bm = np.zeros((H, 3, 3), np.uint8)
    pick = {0: 2, 1: 0, 2: 1}                 # query tile -> its only key tile (same for both heads)
    for i, j in pick.items():
        bm[:, i, j] = 1
    o, lse = oracle.fwd(q, k, v, 0.7, False, block_mask=bm, block=blk)
    for i, j in pick.items():
        qs = q[:, :, i * blk:(i + 1) * blk]
        ks, vs = k[:, :, j * blk:(j + 1) * blk], v[:, :, j * blk:(j + 1) * blk]
        o2, l2 = oracle.fwd(qs, ks, vs, 0.7, False)
        np.testing.assert_allclose(o[:, :, i * blk:(i + 1) * blk], o2, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[:, :, i * blk:(i + 1) * blk], l2, rtol=0, atol=1e-13)


def test_block_mask_lower_triangle_with_causal_is_causal():
    B, H, N, d, blk = 1, 2, 10, 4, 3
    q, k, v, do = (rnd((B, H, N, d), s) for s in (71, 72, 73, 74))
    nb = -(-N // blk)
    tri = np.tril(np.ones((nb, nb), np.uint8))[None].repeat(H, 0)
    ones = np.ones((H, nb, nb), np.uint8)
    for bm in (tri, ones):
        a = oracle.fwd(q, k, v, 0.5, True, block_mask=bm, block=blk)
        b = oracle.fwd(q, k, v, 0.5, True)
        for x, y in zip(a, b):
            np.testing.assert_array_equal(x, y)
        ga = oracle.bwd(q, k, v, do, 0.5, True, block_mask=bm, block=blk)
        gb = oracle.bwd(q, k, v, do, 0.5, True)
        for x, y in zip(ga, gb):
            np.testing.assert_array_equal(x, y)


def test_block_mask_finite_differences():
    B, H, N, d, blk = 1, 1, 8, 3, 2
    q, k, v, G = (rnd((B, H, N, d), s) for s in (81, 82, 83, 84))
    bm = _tile_mask(H, N // blk, 85)
    bm[0, 2, :] = 0
    bm[0, 0, 0] = 1
    scale = 0.8

    def loss(qq, kk, vv):
        o, _ = oracle.fwd(qq, kk, vv, scale, True, block_mask=bm, block=blk)
        return float(np.sum(o * G))

    dq, dk, dv = oracle.bwd(q, k, v, G, scale, True, block_mask=bm, block=blk)
    h = 1e-6
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = x.copy(); xp[idx] += h
            xm = x.copy(); xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        err = np.max(np.abs(num - grad)) / max(1e-12, np.max(np.abs(grad)))
        assert err < 1e-6, (name, err)


def test_block_mask_rejected_with_packed_layout():
    q = np.zeros((8, 1, 4))
    with pytest.raises(ValueError):
        oracle.fwd(q, q, q, 1.0, False, cu_seqlens=[0, 3, 8], block_mask=np.ones((1, 1, 1), np.uint8), block=128)


# ---------------------------------------------------------------- e4m3 (FP8) inputs
def test_e4m3_decode_closed_forms():
    # values fixed by the format: sign bit, 4-bit exponent with bias 7, 3-bit mantissa,
    # subnormals at exponent 0, NaN only at S.1111.111, no infinities
    want = {0x00: 0.0, 0x38: 1.0, 0x3C: 1.5, 0x40: 2.0, 0x30: 0.5, 0x7E: 448.0, 0x77: 240.0,
            0x08: 2.0 ** -6, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x0F: 1.875 * 2.0 ** -6,
            0xB8: -1.0, 0xFE: -448.0, 0x81: -(2.0 ** -9), 0x7D: 416.0, 0x78: 256.0}
    codes = np.array(sorted(want), dtype=np.uint8)
    got = oracle.e4m3_decode(codes)
    assert list(got) == [want[c] for c in sorted(want)]
    z = oracle.e4m3_decode(np.array([0x80], dtype=np.uint8))
    assert z[0] == 0.0 and math.copysign(1.0, z[0]) == -1.0  # negative zero
    nan = oracle.e4m3_decode(np.array([0x7F, 0xFF], dtype=np.uint8))
    assert np.isnan(nan).all()


def test_e4m3_decode_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    lib_vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(oracle.e4m3_decode(codes), lib_vals, equal_nan=True)
    # finite codes are strictly increasing in magnitude with the code, sign aside
    pos = oracle.e4m3_decode(codes[:0x7F])
    assert np.all(np.diff(pos) > 0)


def test_e4m3_decode_applies_the_factor():
    codes = np.arange(0, 0x7F, dtype=np.uint8)
    base = oracle.e4m3_decode(codes)
    for f in (0.25, 3.0, 1.0 / 448.0):
        assert np.array_equal(oracle.e4m3_decode(codes, f), base * f)


def test_fwd_fp8_is_attention_of_the_decoded_inputs():
    # distinct factors per tensor, so a swapped operand or factor shows up
    from attn_inputs import make_fp8
    inp = make_fp8(1, 2, 96, 16, seed=8100, causal=True)
    dec = [torch.from_numpy(t.numpy()).view(torch.float8_e4m3fn).to(torch.float64) * f
           for t, f in ((inp.q8, inp.q_scale), (inp.k8, inp.k_scale), (inp.v8, 3.0 * inp.v_scale))]
    o8, l8 = oracle.fwd_fp8(inp.q8, inp.k8, inp.v8, inp.q_scale, inp.k_scale, 3.0 * inp.v_scale, inp.scale, True)
    o, l = oracle.fwd(dec[0], dec[1], dec[2], inp.scale, True)
    assert np.array_equal(o8, o) and np.array_equal(l8, l)
