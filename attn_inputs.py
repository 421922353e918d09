"""Seeded synthetic inputs shared by the CUDA path's tests/bench and by the CPU oracle.

This module only draws random numbers and builds masks/length tables.  It holds
none of the attention arithmetic, so it can serve both sides without coupling them.

Recipe (one ``torch.Generator('cpu')`` per workload, values drawn in float32 and
rounded to bf16, tensors drawn in the order Q, K, V, dO):

* dense tensors are ``[B, H, N, d]`` row-major;
* packed variable-length tensors are token-major ``[total, H, d]`` with
  ``cu_seqlens[B+1]`` (int32) giving each sequence's first token;
* the key-padding mask ``key_keep`` is uint8, 1 = attend, 0 = masked, shaped
  ``[B, N]`` (dense) or ``[total]`` (packed);
* e4m3 (FP8) inputs are float32 draws for Q, K, V (in that order) quantised per
  tensor the way a caller prepares them: factor = amax / 448, codes from torch's
  ``float8_e4m3fn`` rounding (``make_fp8``, ``make_fp8_varlen``);
* block-sparse tile masks are uint8 ``[H, nb, nb]`` Bernoulli draws (``tile_mask``).

The shapes follow the workloads the attention pages talk about: sequence length
2048 ("PyTorch Attention 层性能分析与优化" / codechina FlashAttention article §5.2
timing table) and the N=4096, d=128 tiling example (codechina article §2.2).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch


@dataclass
class Workload:
    name: str
    seed: int
    B: int
    H: int
    N: int
    d: int
    causal: bool
    qk_sigma: float = 1.0
    varlen: bool = False
    with_key_mask: bool = False
    with_grad: bool = False
    lengths_seed: int = 0
    mask_seed: int = 0
    n_seqs: int = 0
    len_lo: int = 0
    len_hi: int = 0
    notes: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


# The five workload families.  Sizes are the ones the parity tests and the bench use.
WORKLOADS = {
    "tiny": Workload("tiny causal fwd B1 H2 N128 d64", 1, 1, 2, 128, 64, True),
    "n2048_d64": Workload("causal fwd B4 H16 N2048 d64", 2, 4, 16, 2048, 64, True),
    "n4096_d128": Workload("causal fwd B2 H16 N4096 d128", 3, 2, 16, 4096, 128, True),
    "n4096_d128_wide": Workload("causal fwd B2 H16 N4096 d128, Q,K ~ N(0,4^2)", 33, 2, 16, 4096, 128,
                                True, qk_sigma=4.0),
    "varlen": Workload("varlen causal fwd 8 seqs len U[256,4096] H32 d128 + key padding",
                       4, 8, 32, 4096, 128, True, varlen=True, with_key_mask=True,
                       lengths_seed=40, mask_seed=41, n_seqs=8, len_lo=256, len_hi=4096),
    "bwd_n4096_d128": Workload("causal bwd B2 H16 N4096 d128", 5, 2, 16, 4096, 128, True, with_grad=True),
}


def bf16_randn(gen: torch.Generator, shape, sigma: float = 1.0) -> torch.Tensor:
    """float32 N(0, sigma^2) draws rounded to bf16 (round-to-nearest-even)."""
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if sigma != 1.0:
        x = x * sigma
    return x.to(torch.bfloat16)


def draw_lengths(n_seqs: int, lo: int, hi: int, seed: int) -> list[int]:
    g = torch.Generator("cpu").manual_seed(seed)
    return [int(x) for x in torch.randint(lo, hi + 1, (n_seqs,), generator=g)]


def cu_seqlens_of(lengths) -> torch.Tensor:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32)


def padding_key_mask(lengths, seed: int, pad_frac: float = 0.02, extra_frac: float = 0.01) -> torch.Tensor:
    """Packed ``[total]`` uint8 key mask.

    In every sequence the first ceil(pad_frac*n) keys are masked, so under causal
    masking exactly those query rows see no key at all.  A further ``extra_frac`` of
    the keys after the first unpadded one are masked at random; the first unpadded
    key is never masked, so those extra holes never empty a row.
    """
    g = torch.Generator("cpu").manual_seed(seed)
    parts = []
    for n in lengths:
        n = int(n)
        keep = torch.ones(n, dtype=torch.uint8)
        p = min(n, math.ceil(pad_frac * n))
        keep[:p] = 0
        cand = n - p - 1
        if cand > 0:
            k = int(round(extra_frac * n))
            if k > 0:
                idx = torch.randperm(cand, generator=g)[:k] + p + 1
                keep[idx] = 0
        parts.append(keep)
    return torch.cat(parts)


def tile_mask(H: int, N: int, seed: int, density: float = 0.5, tile: int = 128,
              empty_rows=(), empty_cols=()) -> torch.Tensor:
    """uint8 ``[H, nb, nb]`` block-sparse tile mask, nb = ceil(N / tile): each
    (query tile, key tile) pair kept with probability ``density``.  ``empty_rows`` /
    ``empty_cols`` list (h, tile) pairs whose whole mask row / column is cleared
    (a query tile that sees no key / a key tile that no query reaches)."""
    nb = -(-N // tile)
    g = torch.Generator("cpu").manual_seed(seed)
    m = (torch.rand((H, nb, nb), generator=g) < density).to(torch.uint8)
    for h, i in empty_rows:
        m[h, i, :] = 0
    for h, j in empty_cols:
        m[h, :, j] = 0
    return m


@dataclass
class Inputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    do: Optional[torch.Tensor]
    B: int
    H: int
    N: int
    d: int
    scale: float
    causal: bool
    cu_seqlens: Optional[torch.Tensor] = None
    key_keep: Optional[torch.Tensor] = None
    lengths: list = field(default_factory=list)


def make_dense(B, H, N, d, seed, causal=True, qk_sigma=1.0, with_grad=False,
               key_keep: Optional[torch.Tensor] = None, scale: Optional[float] = None) -> Inputs:
    g = torch.Generator("cpu").manual_seed(seed)
    q = bf16_randn(g, (B, H, N, d), qk_sigma)
    k = bf16_randn(g, (B, H, N, d), qk_sigma)
    v = bf16_randn(g, (B, H, N, d))
    do = bf16_randn(g, (B, H, N, d)) if with_grad else None
    return Inputs(q, k, v, do, B, H, N, d, scale if scale is not None else 1.0 / math.sqrt(d),
                  causal, None, key_keep, [N] * B)


def make_varlen(lengths, H, d, seed, causal=True, key_keep=None, with_grad=False,
                scale: Optional[float] = None) -> Inputs:
    total = int(sum(lengths))
    g = torch.Generator("cpu").manual_seed(seed)
    q = bf16_randn(g, (total, H, d))
    k = bf16_randn(g, (total, H, d))
    v = bf16_randn(g, (total, H, d))
    do = bf16_randn(g, (total, H, d)) if with_grad else None
    return Inputs(q, k, v, do, len(lengths), H, max(lengths), d,
                  scale if scale is not None else 1.0 / math.sqrt(d), causal,
                  cu_seqlens_of(lengths), key_keep, list(lengths))


def make_workload(name: str, **over) -> Inputs:
    w = WORKLOADS[name]
    if w.varlen:
        lengths = draw_lengths(w.n_seqs, w.len_lo, w.len_hi, w.lengths_seed)
        keep = padding_key_mask(lengths, w.mask_seed) if w.with_key_mask else None
        return make_varlen(lengths, w.H, w.d, w.seed, w.causal, keep, over.get("with_grad", w.with_grad))
    return make_dense(w.B, w.H, w.N, w.d, w.seed, over.get("causal", w.causal), w.qk_sigma,
                      over.get("with_grad", w.with_grad))


@dataclass
class Fp8Inputs:
    q8: torch.Tensor  # uint8 e4m3 codes [B, H, N, d]
    k8: torch.Tensor
    v8: torch.Tensor
    q_scale: float    # per-tensor dequantisation factors: value = decode(code) * factor
    k_scale: float
    v_scale: float
    B: int
    H: int
    N: int
    d: int
    scale: float
    causal: bool


def e4m3_codes(x: torch.Tensor):
    """Per-tensor e4m3 quantisation of float32 draws, the way a caller prepares FP8
    inputs: factor = amax / 448 (e4m3's largest finite value), codes = x / factor
    rounded by torch's float8_e4m3fn conversion.  Returns (uint8 codes, factor)."""
    amax = float(x.abs().max())
    factor = amax / 448.0 if amax > 0 else 1.0
    return (x / factor).to(torch.float8_e4m3fn).view(torch.uint8), factor


def make_fp8_varlen(lengths, H, d, seed, causal=True, scale: Optional[float] = None):
    """Packed [total, H, d] e4m3 inputs (as ``make_fp8``) and cu_seqlens.  Returns
    (Fp8Inputs with N = max length, cu_seqlens)."""
    total = int(sum(lengths))
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn(total, H, d, generator=g, dtype=torch.float32)
    k = torch.randn(total, H, d, generator=g, dtype=torch.float32)
    v = torch.randn(total, H, d, generator=g, dtype=torch.float32)
    (q8, qs), (k8, ks), (v8, vs) = e4m3_codes(q), e4m3_codes(k), e4m3_codes(v)
    inp = Fp8Inputs(q8, k8, v8, qs, ks, vs, len(lengths), H, max(lengths), d,
                    scale if scale is not None else 1.0 / math.sqrt(d), causal)
    return inp, cu_seqlens_of(lengths)


def make_fp8(B, H, N, d, seed, causal=True, qk_sigma=1.0, scale: Optional[float] = None) -> Fp8Inputs:
    """N(0, sigma^2) float32 draws for Q, K (sigma = qk_sigma) and V (sigma 1), in
    that order, each quantised per tensor with ``e4m3_codes``."""
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn(B, H, N, d, generator=g, dtype=torch.float32) * qk_sigma
    k = torch.randn(B, H, N, d, generator=g, dtype=torch.float32) * qk_sigma
    v = torch.randn(B, H, N, d, generator=g, dtype=torch.float32)
    (q8, qs), (k8, ks), (v8, vs) = e4m3_codes(q), e4m3_codes(k), e4m3_codes(v)
    return Fp8Inputs(q8, k8, v8, qs, ks, vs, B, H, N, d, scale if scale is not None else 1.0 / math.sqrt(d), causal)

