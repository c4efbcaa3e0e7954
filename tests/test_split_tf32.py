"""The error model of the split-tf32 products that compute the predictor's logits (csrc/score.cuh).

Each fp32 operand x is split into hi = x rounded to tf32 (10 explicit mantissa bits, nearest, ties away
from zero) and lo = x - hi, and a b is taken as hi_a hi_b + hi_a lo_b + lo_a hi_b, the tensor cores seeing
lo only to tf32 precision. This file checks, in float64 on the host, the bound the kernel's header states
(what is left out is under 1.25 x 2^-20 |a b| per product) with lo cut to tf32 by truncation (the worse
case), and that dot products of the predictor's lengths land as close to the float64 result as an fp32
dot product does. No device code runs here; the kernel itself is compared with the oracle by the GPU
parity tests.
"""
import numpy as np
import pytest

TF32_MASK = np.uint32(0xFFFFE000)


def round_tf32(x):
    """x (float32) to the nearest tf32 value, ties away from zero, as float32."""
    b = x.astype(np.float32).view(np.uint32)
    return ((b + np.uint32(0x1000)) & TF32_MASK).view(np.float32)


def trunc_tf32(x):
    return (x.astype(np.float32).view(np.uint32) & TF32_MASK).view(np.float32)


def split(x):
    hi = round_tf32(x)
    lo = (x - hi).astype(np.float32)  # exact: hi and x share their top bits
    return hi, lo


def split_product(a, b):
    ah, al = split(a)
    bh, bl = split(b)
    al, bl = trunc_tf32(al).astype(np.float64), trunc_tf32(bl).astype(np.float64)
    ah, bh = ah.astype(np.float64), bh.astype(np.float64)
    return ah * bh + ah * bl + al * bh


def test_split_is_exact_and_small():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(200_000) * np.exp2(rng.integers(-30, 30, 200_000))).astype(np.float32)
    hi, lo = split(x)
    assert np.all((hi.view(np.uint32) & ~TF32_MASK) == 0)  # hi is a tf32 value
    assert np.array_equal(hi.astype(np.float64) + lo.astype(np.float64), x.astype(np.float64))  # exact
    assert np.all(np.abs(lo.astype(np.float64)) <= np.exp2(-11) * np.abs(x.astype(np.float64)))


def test_ties_round_away_from_zero():
    # 1 + 2^-11 lies halfway between the tf32 neighbours 1 and 1 + 2^-10
    x = np.array([1 + 2.0 ** -11, -(1 + 2.0 ** -11), 1 + 2.0 ** -11 - 2.0 ** -23], np.float32)
    assert round_tf32(x).tolist() == [1 + 2.0 ** -10, -(1 + 2.0 ** -10), 1.0]


def test_per_product_bound():
    rng = np.random.default_rng(11)
    a = (rng.standard_normal(500_000) * np.exp2(rng.integers(-20, 20, 500_000))).astype(np.float32)
    b = (rng.standard_normal(500_000) * np.exp2(rng.integers(-20, 20, 500_000))).astype(np.float32)
    exact = a.astype(np.float64) * b.astype(np.float64)
    rel = np.abs(split_product(a, b) - exact) / np.abs(exact)
    assert rel.max() <= 1.25 * np.exp2(-20)
    # the bound is not loose by orders of magnitude: the largest relative error is within 8x of it
    assert rel.max() > 1.25 * np.exp2(-20) / 8


@pytest.mark.parametrize("k", [128, 384])
def test_dot_products_as_close_as_fp32(k):
    # the predictor's lengths (logits: D = 128; projections: 3D = 384), 2,000 rows of N(0, 1) features
    rng = np.random.default_rng(k)
    a = rng.standard_normal((2000, k)).astype(np.float32)
    b = rng.standard_normal((2000, k)).astype(np.float32)
    exact = (a.astype(np.float64) * b.astype(np.float64)).sum(1)
    scale = (np.abs(a.astype(np.float64)) * np.abs(b.astype(np.float64))).sum(1)
    split_err = np.abs(split_product(a, b).sum(1) - exact) / scale
    fp32 = np.zeros(2000, np.float32)
    for j in range(k):  # an fp32 dot product in order, one rounding per multiply-add
        fp32 = (fp32.astype(np.float64) + a[:, j].astype(np.float64) * b[:, j].astype(np.float64)).astype(np.float32)
    fp32_err = np.abs(fp32.astype(np.float64) - exact) / scale
    # the split's products are below fp32's own rounding: its worst case stays within that of fp32
    assert split_err.max() <= fp32_err.max()
    assert split_err.max() <= 1.25 * np.exp2(-20)
