"""Forward parity: the sm_100a kernel (through the C ABI) against the float64 CPU
oracle on the same seeded bf16 inputs.

Tolerances: O (bf16)  |err| <= 1e-2 + 1e-2 |ref|  elementwise;
            lse (fp32) |err| <= 1e-3, and exactly -inf where the oracle has -inf.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from attn_inputs import make_dense, make_varlen, make_workload, padding_key_mask

pytestmark = pytest.mark.gpu

O_ATOL, O_RTOL, LSE_ATOL = 1e-2, 1e-2, 1e-3


@pytest.fixture(scope="module")
def ea():
    from exact_attention_123_b200 import build
    build.build()
    import exact_attention_123_b200 as m
    assert torch.cuda.is_available()
    return m


def assert_o(got, ref, mask=None, what="O"):
    got = got.detach().cpu().to(torch.float64).numpy()
    if mask is not None:
        got, ref = got[mask], ref[mask]
    assert not np.any(np.isnan(got)), f"{what}: NaN in GPU output"
    err = np.abs(got - ref)
    bad = err > O_ATOL + O_RTOL * np.abs(ref)
    if bad.any():
        i = np.unravel_index(np.argmax(err - O_RTOL * np.abs(ref)), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; worst at {i}: "
                             f"gpu {got[i]} ref {ref[i]}")


def assert_lse(got, ref, mask=None):
    got = got.detach().cpu().to(torch.float64).numpy()
    if mask is not None:
        got, ref = got[mask], ref[mask]
    ninf = np.isneginf(ref)
    assert np.all(np.isneginf(got[ninf])), "rows with no visible key must have lse = -inf"
    fin = ~ninf
    assert np.all(np.isfinite(got[fin])), "lse must be finite where the oracle's is"
    err = np.abs(got[fin] - ref[fin])
    assert err.size == 0 or err.max() <= LSE_ATOL, f"lse max err {err.max()}"


def gpu_fwd(ea, inp, causal=None, key_keep=None, exact_total=True):
    causal = inp.causal if causal is None else causal
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    o = torch.full_like(q, float("nan"))
    if inp.cu_seqlens is None:
        lse = torch.full(q.shape[:3], float("nan"), device="cuda")
        kk = None if key_keep is None else key_keep.cuda()
        ea.attn_fwd(q, k, v, o, lse, scale=inp.scale, causal=causal, key_keep=kk)
    else:
        lse = torch.full(q.shape[:2], float("nan"), device="cuda")
        kk = None if key_keep is None else key_keep.cuda()
        ea.attn_fwd(q, k, v, o, lse, scale=inp.scale, causal=causal, cu_seqlens=inp.cu_seqlens.cuda(),
                    key_keep=kk, max_seqlen=inp.N)
    assert ea.attn_status() == ea.ATTN_OK
    return o, lse


def test_tiny_causal(ea):
    inp = make_workload("tiny")
    o, lse = gpu_fwd(ea, inp)
    ro, rl = oracle.fwd(inp.q, inp.k, inp.v, inp.scale, True)
    assert_o(o, ro)
    assert_lse(lse, rl)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 5, 127, 128, 129, 300, 513])
@pytest.mark.parametrize("causal", [True, False])
def test_dense_shapes(ea, d, N, causal):
    inp = make_dense(2, 3, N, d, seed=1000 + N + d, causal=causal)
    o, lse = gpu_fwd(ea, inp)
    ro, rl = oracle.fwd(inp.q, inp.k, inp.v, inp.scale, causal)
    assert_o(o, ro)
    assert_lse(lse, rl)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
def test_dense_key_mask(ea, d, causal):
    B, N = 2, 300
    inp = make_dense(B, 2, N, d, seed=2000 + d)
    g = torch.Generator().manual_seed(7)
    keep = (torch.rand(B, N, generator=g) > 0.1).to(torch.uint8)
    keep[:, :3] = 0          # causal: rows 0..2 see nothing
    keep[1, 128:256] = 0     # a whole key tile masked
    o, lse = gpu_fwd(ea, inp, causal=causal, key_keep=keep)
    ro, rl = oracle.fwd(inp.q, inp.k, inp.v, inp.scale, causal, key_keep=keep)
    assert_o(o, ro)
    assert_lse(lse, rl)
    if causal:
        assert torch.all(o[:, :, :3].float().cpu() == 0)


@pytest.mark.parametrize("d", [64, 128])
def test_all_keys_masked_gives_zero_not_nan(ea, d):
    inp = make_dense(1, 2, 200, d, seed=3000)
    keep = torch.zeros(1, 200, dtype=torch.uint8)
    for causal in (True, False):
        o, lse = gpu_fwd(ea, inp, causal=causal, key_keep=keep)
        assert torch.all(o.float().cpu() == 0)
        assert torch.all(torch.isneginf(lse.cpu()))


@pytest.mark.parametrize("d", [64, 128])
def test_wide_scores_rescaling(ea, d):
    # Q, K ~ N(0, 4^2): scaled scores spread over tens of units, so the running
    # max moves often and the lazy correction path is exercised.
    inp = make_dense(1, 4, 700, d, seed=4000 + d, qk_sigma=4.0)
    for causal in (True, False):
        o, lse = gpu_fwd(ea, inp, causal=causal)
        ro, rl = oracle.fwd(inp.q, inp.k, inp.v, inp.scale, causal)
        assert_o(o, ro)
        assert_lse(lse, rl)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
def test_varlen_packed(ea, d, causal):
    lengths = [1, 130, 257, 64, 300, 128]
    inp = make_varlen(lengths, 3, d, seed=5000 + d)
    keep = padding_key_mask(lengths, seed=5001, pad_frac=0.05, extra_frac=0.05)
    o, lse = gpu_fwd(ea, inp, causal=causal, key_keep=keep)
    ro, rl = oracle.fwd(inp.q, inp.k, inp.v, inp.scale, causal, cu_seqlens=inp.cu_seqlens, key_keep=keep)
    assert_o(o, ro)
    assert_lse(lse, rl)


def test_varlen_guard_band_untouched(ea):
    # Output rows past the packed tokens must stay as they were (NaN sentinel):
    # tail tiles of the last sequence must not be stored.
    lengths = [70, 200]
    inp = make_varlen(lengths, 2, 128, seed=5100)
    total = sum(lengths)
    pad = 300
    q = torch.zeros(total + pad, 2, 128, dtype=torch.bfloat16)
    k, v = q.clone(), q.clone()
    q[:total], k[:total], v[:total] = inp.q, inp.k, inp.v
    o = torch.full((total + pad, 2, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((total + pad, 2), float("nan"), device="cuda")
    # exact total: only `total` rows are described to the tile loader
    ea.attn_fwd(q[:total].cuda(), k[:total].cuda(), v[:total].cuda(), o[:total], lse[:total], scale=inp.scale,
                causal=True, cu_seqlens=inp.cu_seqlens.cuda(), max_seqlen=max(lengths))
    assert ea.attn_status() == 0
    assert torch.all(torch.isnan(o[total:].float()))
    assert torch.all(torch.isnan(lse[total:]))
    ro, rl = oracle.fwd(inp.q, inp.k, inp.v, inp.scale, True, cu_seqlens=inp.cu_seqlens)
    assert_o(o[:total], ro)
    assert_lse(lse[:total], rl)


def test_varlen_through_padded_entry_point(ea):
    # attn_fwd with cu_seqlens assumes the packed buffers span B*N rows.
    lengths = [100, 37, 256]
    B, N, H, d = len(lengths), 260, 2, 64
    inp = make_varlen(lengths, H, d, seed=5200)
    total = sum(lengths)
    q = torch.zeros(B * N, H, d, dtype=torch.bfloat16)
    k, v = q.clone(), q.clone()
    q[:total], k[:total], v[:total] = inp.q, inp.k, inp.v
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o = torch.full_like(qc, float("nan"))
    lse = torch.full((B * N, H), float("nan"), device="cuda")
    L = ea.lib()
    import ctypes
    rc = L.attn_fwd(ctypes.c_void_p(qc.data_ptr()), ctypes.c_void_p(kc.data_ptr()), ctypes.c_void_p(vc.data_ptr()),
                    ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()), B, H, N, d,
                    ctypes.c_float(inp.scale), 1, ctypes.c_void_p(inp.cu_seqlens.cuda().data_ptr()),
                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0 and ea.attn_status() == 0
    ro, rl = oracle.fwd(inp.q, inp.k, inp.v, inp.scale, True, cu_seqlens=inp.cu_seqlens)
    assert_o(o[:total], ro)
    assert_lse(lse[:total], rl)
    assert torch.all(torch.isnan(o[total:].float()))


# ------------------------------------------------------------------ full-size workloads, sampled slices

def sampled(inp, picks):
    BH = inp.B * inp.H
    return sorted({p % BH for p in picks})


@pytest.mark.parametrize("name,causal", [("n2048_d64", True), ("n2048_d64", False), ("n4096_d128", True),
                                         ("n4096_d128", False), ("n4096_d128_wide", True),
                                         ("n4096_d128_wide", False)])
def test_full_size_sampled(ea, name, causal):
    inp = make_workload(name, causal=causal)
    o, lse = gpu_fwd(ea, inp, causal=causal)
    sl = sampled(inp, [0, 7, inp.B * inp.H - 1])
    ro, rl = oracle.fwd(inp.q, inp.k, inp.v, inp.scale, causal, slices=sl)
    B, H = inp.B, inp.H
    for s in sl:
        b, h = divmod(s, H)
        assert_o(o[b, h], ro[b, h], what=f"O slice {s}")
        assert_lse(lse[b, h], rl[b, h])
    assert not torch.isnan(o.float()).any()


def test_full_size_varlen_sampled(ea):
    inp = make_workload("varlen")
    o, lse = gpu_fwd(ea, inp, key_keep=inp.key_keep)
    H = inp.H
    picks = [0 * H + 0, 3 * H + 17, (inp.B - 1) * H + H - 1]
    ro, rl = oracle.fwd(inp.q, inp.k, inp.v, inp.scale, True, cu_seqlens=inp.cu_seqlens, key_keep=inp.key_keep,
                        slices=picks)
    cu = inp.cu_seqlens.tolist()
    for s in picks:
        b, h = divmod(s, H)
        rows = slice(cu[b], cu[b + 1])
        assert_o(o[rows, h], ro[rows, h], what=f"O seq {b} head {h}")
        assert_lse(lse[rows, h], rl[rows, h])
        n = cu[b + 1] - cu[b]
        p = math.ceil(0.02 * n)
        assert torch.all(o[cu[b]:cu[b] + p, h].float().cpu() == 0)          # padded rows: 0, not NaN
        assert torch.all(torch.isneginf(lse[cu[b]:cu[b] + p, h].cpu()))
    assert not torch.isnan(o.float()).any()


def test_binding_rejects_mismatched_buffers(ea):
    # The C ABI takes raw pointers with sizes; the binding checks every tensor's shape,
    # dtype and device first, so no kernel ever sees a buffer smaller than its sizes.
    dev = "cuda"
    q = torch.zeros(1, 2, 256, 64, device=dev, dtype=torch.bfloat16)
    small = torch.zeros(1, 2, 128, 64, device=dev, dtype=torch.bfloat16)
    lse = torch.zeros(1, 2, 256, device=dev)
    cases = [
        lambda: ea.attn_fwd(q, small, q),                                     # k shorter than q
        lambda: ea.attn_fwd(q, q, q, small),                                  # o too small
        lambda: ea.attn_fwd(q, q, q, None, torch.zeros(1, 2, 128, device=dev)),  # lse too small
        lambda: ea.attn_fwd(q, q, q.float()),                                 # v not bf16
        lambda: ea.attn_fwd(q, q, q, key_keep=torch.ones(1, 255, device=dev, dtype=torch.uint8)),
        lambda: ea.attn_fwd(q[0], q[0], q[0]),                                # not 4-D
        lambda: ea.attn_bwd(q, q, q, q, lse, small),                          # dO too small
        lambda: ea.attn_bwd(q, q, q, q, lse, q, small),                       # dQ too small
        lambda: ea.attn_bwd(q, q, q, q, torch.zeros(2, 256, device=dev), q),  # lse shape
        lambda: ea.attn_bwd_noalloc(q, q, q, q, lse, q, None, small),         # dK too small
        lambda: ea.attn_fwd_blocksparse(q, q, q, torch.ones(2, 1, 1, device=dev, dtype=torch.uint8)),
        lambda: ea.attn_fwd_fp8(q.view(torch.uint8)[..., :64].contiguous(), q, q, 1.0, 1.0, 1.0),
    ]
    for i, call in enumerate(cases):
        with pytest.raises(ValueError):
            call()
            pytest.fail(f"case {i} was accepted")
    assert ea.attn_status() == ea.ATTN_OK
