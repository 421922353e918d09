"""FP8 (e4m3) forward parity: the sm_100a kernel through the C ABI against the
float64 oracle's attention of the decoded inputs.

Tolerance, derived from the kernel's arithmetic.  Q K^T and P V take e4m3 operands
with fp32 accumulation; the one rounding beyond the bf16 path's is P, rounded to
e4m3 on a scale where the row's running maximum is at most 2^8 (lazy rescaling)
and the row sum is at least the true one (the running maximum never exceeds the
true maximum).  Round-to-nearest e4m3 errs by at most 2^-4 of a normal value and
by 2^-10 absolute below 2^-6.  The probabilities themselves carry the relative
error eps of the exponential (1.02e-4 for the eighth computed by the cubic on the
FMA pipe, 2^-22 for the MUFU ones), so each weight w_ij = softmax_j of the
rounded P errs by at most
    e_ij = max((2^-4 + 2^-12) w_ij, 2^-10 / l'_i),  l'_i = sum_j exp(S_ij - max_j S_ij)
(0 for masked keys; 2^-12 > eps (1 + 2^-4)), and the output element by
sum_j e_ij |V_jc|.  The row sum, made of the unrounded probabilities, carries eps
too: O moves by at most eps |O_ic| (taken as 2^-13).  On top: bf16 rounding of O
(2^-8 relative), and an allowance of 1e-3 on every score for the fp32 (or
narrower) accumulation of the e4m3 products, which moves O by at most
1e-3 (sum_j w_ij |V_jc| + |O_ic|).  lse: |err| <= 1e-3 (scores and eps).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from attn_inputs import make_fp8

pytestmark = pytest.mark.gpu

LSE_ATOL = 1e-3
S_ALLOW = 1e-3


@pytest.fixture(scope="module")
def ea():
    from exact_attention_123_b200 import build
    build.build()
    import exact_attention_123_b200 as m
    assert torch.cuda.is_available()
    return m


def gpu_fp8(ea, inp, causal=None, key_keep=None, cu_seqlens=None):
    causal = inp.causal if causal is None else causal
    q8, k8, v8 = inp.q8.cuda(), inp.k8.cuda(), inp.v8.cuda()
    o = torch.full(q8.shape, float("nan"), device="cuda", dtype=torch.bfloat16)
    lse = torch.full(q8.shape[:2] if cu_seqlens is not None else q8.shape[:3], float("nan"), device="cuda")
    kw = {}
    if cu_seqlens is not None:
        kw = dict(cu_seqlens=cu_seqlens.cuda(), max_seqlen=inp.N)
    ea.attn_fwd_fp8(q8, k8, v8, inp.q_scale, inp.k_scale, inp.v_scale, o, lse, scale=inp.scale, causal=causal,
                    key_keep=None if key_keep is None else key_keep.cuda(), **kw)
    assert ea.attn_status() == ea.ATTN_OK
    return o.double().cpu().numpy(), lse.double().cpu().numpy()


def bound_slice(qd, kd, vd, scale, causal, o_ref, lse_ref, keep=None, pairs=None):
    """Elementwise error bound for one (sequence, head) slice (float64 numpy, n x d),
    over the rows that see at least one key (the others are checked exactly).
    ``pairs``: n x n booleans, the (query, key) pairs a tile mask keeps."""
    n = qd.shape[0]
    S = scale * (qd @ kd.T)
    if causal:
        S[np.triu_indices(n, 1)] = -np.inf
    if keep is not None:
        S[:, ~keep] = -np.inf
    if pairs is not None:
        S[~pairs] = -np.inf
    live = np.isfinite(lse_ref)
    S, o_l, lse_l = S[live], o_ref[live], lse_ref[live]
    m = S.max(axis=1)
    W = np.exp(S - lse_l[:, None])
    lp = np.exp(lse_l - m)
    E = np.where(np.isfinite(S), np.maximum((2.0 ** -4 + 2.0 ** -12) * W, (2.0 ** -10 / lp)[:, None]), 0.0)
    A = np.abs(vd)
    tol = np.zeros_like(o_ref)
    tol[live] = E @ A + S_ALLOW * (W @ A + np.abs(o_l)) + (2.0 ** -8 + 2.0 ** -13) * np.abs(o_l) + 1e-6
    return tol, live


def check_slice(tag, qd, kd, vd, scale, causal, got_o, got_l, ro, rl, keep=None, pairs=None):
    tol, live = bound_slice(qd, kd, vd, scale, causal, ro, rl, keep, pairs)
    assert not np.isnan(got_o).any(), f"NaN in {tag}"
    # rows that see no key: exactly O = 0 and lse = -inf
    assert np.all(got_o[~live] == 0.0) and np.all(np.isneginf(got_l[~live])), f"{tag}: empty rows"
    err = np.abs(got_o - ro)
    bad = (err > tol) & live[:, None]
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(live[:, None], err - tol, -np.inf)), err.shape)
        raise AssertionError(f"{tag}: {bad.sum()} elements out of bound; worst at {i}: gpu {got_o[i]} ref {ro[i]} "
                             f"bound {tol[i]}")
    lerr = np.abs(got_l[live] - rl[live])
    assert lerr.size == 0 or lerr.max() <= LSE_ATOL, f"{tag}: lse err {lerr.max()}"
    return float((err[live] / tol[live]).max()) if live.any() else 0.0


def tile_pairs(bm_h, n):
    """n x n booleans: the (query, key) pairs that one head's tile mask keeps."""
    t = np.arange(n) // 128
    return bm_h[t][:, t] != 0


def check(inp, got_o, got_l, causal, slices=None, key_keep=None, block_mask=None):
    keep = None if key_keep is None else key_keep.numpy().astype(bool)
    bm = None if block_mask is None else block_mask.numpy()
    ro, rl = oracle.fwd_fp8(inp.q8, inp.k8, inp.v8, inp.q_scale, inp.k_scale, inp.v_scale, inp.scale, causal,
                            key_keep=key_keep, slices=slices, block_mask=bm)
    qd = oracle.e4m3_decode(inp.q8, inp.q_scale)
    kd = oracle.e4m3_decode(inp.k8, inp.k_scale)
    vd = oracle.e4m3_decode(inp.v8, inp.v_scale)
    worst = 0.0
    for sidx in (slices if slices is not None else range(inp.B * inp.H)):
        b, h = divmod(int(sidx), inp.H)
        worst = max(worst, check_slice(f"slice {sidx}", qd[b, h], kd[b, h], vd[b, h], inp.scale, causal,
                                       got_o[b, h], got_l[b, h], ro[b, h], rl[b, h],
                                       None if keep is None else keep[b],
                                       None if bm is None else tile_pairs(bm[h], inp.N)))
    return worst


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
def test_fp8_ragged_tiles(ea, causal, d):
    # 5 query tiles: two full 256-row units and a half one; keys end mid-tile too
    inp = make_fp8(1, 2, 640 - 37, d, seed=8200 + d, causal=causal)
    o, l = gpu_fp8(ea, inp)
    check(inp, o, l, causal)


def test_fp8_several_slices_and_short_rows(ea):
    inp = make_fp8(2, 3, 333, 128, seed=8201, causal=False)
    o, l = gpu_fp8(ea, inp)
    check(inp, o, l, False)


@pytest.mark.parametrize("N", [1, 17, 128, 129])
def test_fp8_edge_lengths(ea, N):
    inp = make_fp8(1, 1, N, 128, seed=8210 + N, causal=True)
    o, l = gpu_fp8(ea, inp)
    check(inp, o, l, True)


@pytest.mark.parametrize("d", [64, 128])
def test_fp8_wide_scores_exercise_rescaling(ea, d):
    # Q, K ~ N(0, 4^2): scores spread over tens of units, so running maxima move by
    # more than the lazy-rescale threshold and P values reach far below 2^-6
    inp = make_fp8(1, 2, 512, d, seed=8220 + d, causal=True, qk_sigma=4.0)
    o, l = gpu_fp8(ea, inp)
    check(inp, o, l, True)


def test_fp8_bound_is_not_vacuous(ea):
    # the rounding bound must be tight enough to catch a wrong P: the observed error
    # uses a sizeable part of it, but nowhere near all of it
    inp = make_fp8(1, 2, 512, 128, seed=8230, causal=True)
    o, l = gpu_fp8(ea, inp)
    worst = check(inp, o, l, True)
    assert 0.01 < worst <= 1.0


def test_fp8_zero_inputs(ea):
    inp = make_fp8(1, 1, 200, 128, seed=8240, causal=True)
    z = torch.zeros_like(inp.q8)
    inp.q8, inp.k8, inp.v8 = z, z.clone(), z.clone()
    o, l = gpu_fp8(ea, inp)
    assert np.all(o == 0.0)
    # all scores 0: row i sees i+1 equal keys
    assert np.allclose(l[0, 0], np.log(np.arange(1, 201)), atol=1e-5)


def test_fp8_repeat_is_bit_identical(ea):
    inp = make_fp8(1, 2, 300, 128, seed=8250, causal=True)
    o1, l1 = gpu_fp8(ea, inp)
    o2, l2 = gpu_fp8(ea, inp)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)  # deterministic
    check(inp, o1, l1, True)


@pytest.mark.parametrize("causal", [True, False])
def test_fp8_full_size_sampled_slices(ea, causal):
    # the benchmark shape (B2 H16 N4096 d128), checked on sampled slices
    inp = make_fp8(2, 16, 4096, 128, seed=8260 + int(causal), causal=causal)
    o, l = gpu_fp8(ea, inp)
    check(inp, o, l, causal, slices=[0, 13, 31])


def test_fp8_dense_key_mask_with_empty_rows(ea):
    # the first 40 keys of sequence 0 are padding: under causal masking its first 40
    # query rows see no key (O = 0, lse = -inf); a scattering of other keys is masked
    from attn_inputs import make_fp8
    inp = make_fp8(2, 2, 300, 128, seed=8270, causal=True)
    g = torch.Generator("cpu").manual_seed(8271)
    keep = (torch.rand(2, 300, generator=g) > 0.1).to(torch.uint8)
    keep[0, :40] = 0
    keep[1, 0] = 1
    o, l = gpu_fp8(ea, inp, key_keep=keep)
    check(inp, o, l, True, key_keep=keep)
    assert np.all(o[0, :, :40] == 0.0) and np.all(np.isneginf(l[0, :, :40]))


@pytest.mark.parametrize("causal", [True, False])
def test_fp8_varlen_with_padding_mask(ea, causal):
    from attn_inputs import make_fp8_varlen, padding_key_mask
    lengths = [300, 129, 1, 517, 128]
    inp, cu = make_fp8_varlen(lengths, 2, 128, seed=8280, causal=causal)
    keep = padding_key_mask(lengths, seed=8281)
    o, l = gpu_fp8(ea, inp, key_keep=keep, cu_seqlens=cu)
    ro, rl = oracle.fwd_fp8(inp.q8, inp.k8, inp.v8, inp.q_scale, inp.k_scale, inp.v_scale, inp.scale, causal,
                            cu_seqlens=cu, key_keep=keep, N=inp.N)
    qd = oracle.e4m3_decode(inp.q8, inp.q_scale)
    kd = oracle.e4m3_decode(inp.k8, inp.k_scale)
    vd = oracle.e4m3_decode(inp.v8, inp.v_scale)
    kp = keep.numpy().astype(bool)
    cuv = cu.tolist()
    for b in range(len(lengths)):
        st, en = cuv[b], cuv[b + 1]
        for h in range(2):
            check_slice(f"seq {b} head {h}", qd[st:en, h], kd[st:en, h], vd[st:en, h], inp.scale, causal,
                        o[st:en, h], l[st:en, h], ro[st:en, h], rl[st:en, h], kp[st:en])


@pytest.mark.parametrize("N", [1, 129])
def test_fp8_d64_edge_lengths(ea, N):
    inp = make_fp8(1, 1, N, 64, seed=8290 + N, causal=True)
    o, l = gpu_fp8(ea, inp)
    check(inp, o, l, True)


def test_fp8_d64_full_size_sampled_slices(ea):
    # the pages' sequence length at d = 64 (causal, B4 H16 N2048), sampled slices
    inp = make_fp8(4, 16, 2048, 64, seed=8295, causal=True)
    o, l = gpu_fp8(ea, inp)
    check(inp, o, l, True, slices=[0, 37, 63])


def test_fp8_d64_varlen_with_padding_mask(ea):
    from attn_inputs import make_fp8_varlen, padding_key_mask
    lengths = [300, 1, 517, 129]
    inp, cu = make_fp8_varlen(lengths, 2, 64, seed=8296, causal=True)
    keep = padding_key_mask(lengths, seed=8297)
    o, l = gpu_fp8(ea, inp, key_keep=keep, cu_seqlens=cu)
    ro, rl = oracle.fwd_fp8(inp.q8, inp.k8, inp.v8, inp.q_scale, inp.k_scale, inp.v_scale, inp.scale, True,
                            cu_seqlens=cu, key_keep=keep, N=inp.N)
    qd = oracle.e4m3_decode(inp.q8, inp.q_scale)
    kd = oracle.e4m3_decode(inp.k8, inp.k_scale)
    vd = oracle.e4m3_decode(inp.v8, inp.v_scale)
    kp = keep.numpy().astype(bool)
    cuv = cu.tolist()
    for b in range(len(lengths)):
        st, en = cuv[b], cuv[b + 1]
        for h in range(2):
            check_slice(f"seq {b} head {h}", qd[st:en, h], kd[st:en, h], vd[st:en, h], inp.scale, True,
                        o[st:en, h], l[st:en, h], ro[st:en, h], rl[st:en, h], kp[st:en])



# ---- FP8 with a block-sparse tile mask (attn_fwd_fp8_blocksparse): the same bound, with
# the pairs the mask leaves out counted as masked scores.

def gpu_fp8_sparse(ea, inp, bm, causal):
    q8, k8, v8 = inp.q8.cuda(), inp.k8.cuda(), inp.v8.cuda()
    o = torch.full(q8.shape, float("nan"), device="cuda", dtype=torch.bfloat16)
    lse = torch.full(q8.shape[:3], float("nan"), device="cuda")
    ea.attn_fwd_fp8_blocksparse(q8, k8, v8, inp.q_scale, inp.k_scale, inp.v_scale, bm.cuda(), o, lse,
                                scale=inp.scale, causal=causal)
    assert ea.attn_status() == ea.ATTN_OK
    return o.double().cpu().numpy(), lse.double().cpu().numpy()


SPARSE_CASES = [
    # B, H, N, d, causal, density, seed, emptied (head, query tile) rows: query tiles
    # with no key tile (first, last and neighbouring tiles), and a ragged N that ends
    # the last tile mid-way.
    (2, 3, 700, 128, False, 0.5, 9301, [(0, 2), (1, 1), (2, 2), (2, 3)]),
    (2, 3, 700, 128, True, 0.6, 9302, [(0, 4), (1, 1)]),
    (1, 4, 1024, 64, False, 0.3, 9303, [(3, 6), (3, 7), (0, 0)]),
    (1, 2, 640, 64, True, 0.5, 9304, [(1, 3), (0, 4)]),
]


@pytest.mark.parametrize("B,H,N,d,causal,density,seed,er", SPARSE_CASES)
def test_fp8_blocksparse_matches_oracle(ea, B, H, N, d, causal, density, seed, er):
    from attn_inputs import tile_mask
    inp = make_fp8(B, H, N, d, seed=seed, causal=causal)
    bm = tile_mask(H, N, seed + 1, density, empty_rows=er)
    o, l = gpu_fp8_sparse(ea, inp, bm, causal)
    check(inp, o, l, causal, block_mask=bm)
    for h, i in er:  # emptied query tiles: O = 0 and lse = -inf exactly
        rows = slice(i * 128, min(N, (i + 1) * 128))
        assert np.all(o[:, h, rows] == 0.0) and np.all(np.isneginf(l[:, h, rows]))


@pytest.mark.parametrize("d,causal", [(128, True), (128, False), (64, False)])
def test_fp8_full_mask_is_the_dense_fp8_path(ea, d, causal):
    # every pair kept: the masked kernel (one query tile per CTA) does the dense e4m3
    # kernel's arithmetic in the same key-tile order, so O and lse match bit for bit (at
    # d = 64 the dense causal kernel sweeps a unit's second tile from its diagonal
    # tile, another order)
    inp = make_fp8(2, 2, 520, d, seed=9310 + d, causal=causal)
    bm = torch.ones((2, 5, 5), dtype=torch.uint8)
    o, l = gpu_fp8_sparse(ea, inp, bm, causal)
    o2, l2 = gpu_fp8(ea, inp, causal=causal)
    assert np.array_equal(o, o2) and np.array_equal(l, l2)


def test_fp8_blocksparse_full_size_sampled_slices(ea):
    # the benchmark shape (B2 H16 N4096 d128, causal) with half of the tile pairs left
    # out by a seeded per-head mask, checked on sampled slices
    from attn_inputs import tile_mask
    inp = make_fp8(2, 16, 4096, 128, seed=9320, causal=True)
    bm = tile_mask(16, 4096, 9321, 0.5, empty_rows=[(13, 5)])
    o, l = gpu_fp8_sparse(ea, inp, bm, True)
    check(inp, o, l, True, slices=[0, 13, 31], block_mask=bm)
