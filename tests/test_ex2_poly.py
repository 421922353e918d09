"""The exponential the d = 64 and e4m3 forward kernels take from the FMA pipe for
part of their scores, held to its stated accuracy directly (the attention parity
bands are far wider than it).

2^x = 2^j * q(f), j = rint(x), f = x - j in [-1/2, 1/2], q(f) = 1 + f (a1 + f (a2 + f a3))
with coefficients fitted by Lawson-weighted least squares towards the minimax
relative error; x is clamped to -127 first, where 2^j is built as +0.

CPU: the committed coefficients (read from the kernel header) meet the bound on
[-1/2, 1/2] in exact arithmetic and in float32 Horner evaluation, and the fitting
method itself, rerun here, lands on coefficients of the same quality.
GPU: the kernels' own function (through the attn_debug_ex2_poly test hook) against
float64 2^x over a dense sweep, the clamp, -inf and the integers.
"""
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BOUND = 1.02e-4


def committed_coefficients():
    src = open(os.path.join(ROOT, "exact_attention_123_b200", "csrc", "sm100_ptx.cuh")).read()
    m = re.search(r"kA1 = ([0-9.eE+-]+)f, kA2 = ([0-9.eE+-]+)f, kA3 = ([0-9.eE+-]+)f", src)
    assert m, "coefficients not found in sm100_ptx.cuh"
    return tuple(float(np.float32(float(g))) for g in m.groups())


def rel_err_exact(a, f):
    a1, a2, a3 = a
    q = 1.0 + f * (a1 + f * (a2 + f * a3))
    return np.abs(q / np.exp2(f) - 1.0)


def f32_fma(a, b, c):
    # a*b is exact in float64 for float32 a, b; one rounding to float32 as fma.rn does
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def rel_err_f32(a, f64):
    a1, a2, a3 = (np.float32(x) for x in a)
    f = f64.astype(np.float32)
    one = np.ones_like(f)
    q = f32_fma(f, np.full_like(f, a3), np.full_like(f, a2))
    q = f32_fma(q, f, np.full_like(f, a1))
    q = f32_fma(q, f, one)
    return np.abs(q.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)


def lawson_fit(iters=400):
    """Degree-3 polynomial with q(0) = 1 minimising the largest relative error
    |q(f) / 2^f - 1| on [-1/2, 1/2]: Lawson's iteration (weighted least squares,
    weights multiplied by the pointwise error each round)."""
    f = np.linspace(-0.5, 0.5, 4001)
    e = np.exp2(f)
    A = np.stack([f / e, f ** 2 / e, f ** 3 / e], axis=1)
    b = (e - 1.0) / e
    w = np.full(f.size, 1.0 / f.size)
    for _ in range(iters):
        sw = np.sqrt(w)
        a, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        r = np.abs(A @ a - b)
        w = w * r
        w /= w.sum()
    return tuple(a)


def test_committed_coefficients_meet_the_bound():
    a = committed_coefficients()
    f = np.linspace(-0.5, 0.5, 200001)
    assert rel_err_exact(a, f).max() <= BOUND
    assert rel_err_f32(a, f).max() <= BOUND
    # the cubic is exact at f = 0, so every integer x gives exactly 2^x
    assert rel_err_exact(a, np.array([0.0]))[0] == 0.0


def test_lawson_fit_reproduces_the_committed_quality():
    a_fit = lawson_fit()
    f = np.linspace(-0.5, 0.5, 200001)
    e_fit = rel_err_exact(a_fit, f).max()
    e_com = rel_err_exact(committed_coefficients(), f).max()
    # the committed coefficients are as good as a fresh minimax-directed fit (to 2 %)
    assert e_com <= 1.02 * e_fit
    assert e_fit <= BOUND
    np.testing.assert_allclose(a_fit, committed_coefficients(), rtol=2e-3)


@pytest.mark.gpu
def test_kernel_exponential_against_float64():
    import torch
    from exact_attention_123_b200 import build
    build.build()
    import exact_attention_123_b200 as ea

    sweep = np.linspace(-130.0, 9.0, 1_390_000, dtype=np.float32)
    ints = np.arange(-130, 10, dtype=np.float32)
    special = np.array([-np.inf, -127.0, -126.75, -126.5, -126.49, -1e30, -200.0, 0.0, -0.0, 0.5, -0.5],
                       dtype=np.float32)
    x = np.concatenate([sweep, ints, special])
    if x.size % 2:
        x = np.append(x, np.float32(0.0))
    y = ea.attn_debug_ex2_poly(torch.from_numpy(x).cuda()).cpu().numpy()
    assert ea.attn_status() == ea.ATTN_OK
    x64, y64 = x.astype(np.float64), y.astype(np.float64)
    ref = np.exp2(x64)
    normal = x64 >= -126.5   # j >= -126: 2^j is a normal float and the cubic carries the error
    assert np.all(np.isfinite(y64))
    assert (np.abs(y64[normal] / ref[normal] - 1.0)).max() <= BOUND
    low = x64 <= -127.0      # the clamp: exactly +0 (sign bit clear), -inf included
    assert np.all(y[low] == 0.0) and not np.any(np.signbit(y[low]))
    between = ~normal & ~low  # j = -127 there: 2^j is built as +0 too
    assert np.all((y64[between] >= 0.0) & (y64[between] <= ref[between]))
    on_int = (x64 == np.round(x64)) & (x64 >= -126)
    assert np.array_equal(y64[on_int], np.exp2(x64[on_int]))  # exact powers of two
