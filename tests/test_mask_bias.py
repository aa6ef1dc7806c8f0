"""The bias operands of the attention kernel's extra tensor-core product, emulated on the CPU.

Key columns outside an item's valid range, and the listed tiles of a landmark chunk, are masked
by one more product S += ones . bias^T: the A tile holds bf16 1.0 (0x3F80) everywhere, and the
bias row of a masked column sums to -2^100 (sixteen elements of -2^96 = 0xEF80, or one element of
-2^100 = 0xF180), that of a valid column to +0.  A landmark column's multiplicity term b (log2 c_j
divided by the base-2 softmax scale, so that it is in units of S) is carried as three bf16 parts
b0 = rn(b), b1 = rn(b - b0), b2 = rn(b - b0 - b1).  These tests pin the encodings, the accuracy
of the split, and the facts the kernel relies on: a masked score is -2^100 whatever the dot
product, and it yields the same exponential as -inf on the FMA-pipe route (the exponent is clamped
at -125 before the polynomial) - the MUFU route returns +0 for both.
"""
import math

import numpy as np


def bf16_bits_rne(x) -> np.ndarray:
    """f32 -> bf16 bit pattern, round to nearest even (as __float2bfloat16_rn)."""
    b = np.asarray(x, np.float32).reshape(-1).view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    return ((b + 0x7FFF + lsb) >> 16).astype(np.uint16)


def bf16_value(bits) -> np.ndarray:
    return (np.asarray(bits, np.uint32).reshape(-1) << 16).astype(np.uint32).view(np.float32)


def split3(b: np.ndarray):
    """The producer's three-part split, in f32 arithmetic."""
    b = np.asarray(b, np.float32)
    p0 = bf16_bits_rne(b)
    r1 = (b - bf16_value(p0)).astype(np.float32)
    p1 = bf16_bits_rne(r1)
    p2 = bf16_bits_rne((r1 - bf16_value(p1)).astype(np.float32))
    return p0, p1, p2


def test_constant_encodings():
    assert bf16_value(0x3F80)[0] == 1.0
    assert bf16_value(0xEF80)[0] == -(2.0 ** 96)
    assert bf16_value(0xF180)[0] == -(2.0 ** 100)
    # sixteen elements of -2^96 times ones sum exactly to -2^100 in f32
    acc = np.float32(0.0)
    for _ in range(16):
        acc = np.float32(acc + np.float32(1.0) * bf16_value(0xEF80)[0])
    assert acc == np.float32(-(2.0 ** 100))


def test_masked_score_absorbs_any_dot_product():
    # |q . k| for bf16 inputs with d = 64 stays far below 2^75 (half an f32 ulp of 2^100 is 2^76)
    rng = np.random.default_rng(5)
    s = (rng.standard_normal(10000) * 10.0 ** rng.uniform(-3, 20, 10000)).astype(np.float32)
    assert (np.abs(s) < 2.0 ** 75).all()
    masked = (s + np.float32(-(2.0 ** 100))).astype(np.float32)
    assert (masked == np.float32(-(2.0 ** 100))).all()
    # a valid column gains exactly +0
    assert ((s + np.float32(0.0)).astype(np.float32) == s).all()


def test_landmark_term_split_keeps_f32_accuracy():
    scale_log2 = np.float32(math.log2(math.e) / 8.0)  # d = 64
    c = np.arange(1, 129, dtype=np.float64)           # key rows of a 128-row tile
    b2 = np.log2(c).astype(np.float32)
    b = (b2 / scale_log2).astype(np.float32)
    p0, p1, p2 = split3(b)
    recon = bf16_value(p0).astype(np.float64) + bf16_value(p1) + bf16_value(p2)
    err = np.abs(recon - b.astype(np.float64))
    assert (err <= 2.0 ** -24 * np.abs(b.astype(np.float64)) + 1e-30).all()
    # a single bf16 part would not do: errors up to 2^-9 relative
    one = np.abs(bf16_value(p0).astype(np.float64) - b)
    assert one.max() > 1e-3 * np.abs(b).max() / 8


def test_split_on_random_values():
    rng = np.random.default_rng(9)
    b = (rng.standard_normal(100000) * 10.0 ** rng.uniform(-6, 6, 100000)).astype(np.float32)
    p0, p1, p2 = split3(b)
    recon = bf16_value(p0).astype(np.float64) + bf16_value(p1) + bf16_value(p2)
    assert (np.abs(recon - b) <= 2.0 ** -24 * np.abs(b.astype(np.float64))).all()


def exp2_poly_fma_route(x: np.ndarray) -> np.ndarray:
    """The FMA-pipe exponential's handling of its argument up to the polynomial: clamp at -125,
    then split into integer and fraction by the 1.5 * 2^23 trick (f32 arithmetic)."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    return np.stack([n, f])


def test_masked_and_minus_inf_give_the_same_exponential():
    scale_log2 = np.float32(math.log2(math.e) / 8.0)
    for m in (np.float32(-3.5), np.float32(0.0), np.float32(41.25)):
        x_inf = np.float32(-np.inf) * scale_log2 - m
        x_big = (np.float32(-(2.0 ** 100)) * scale_log2 - m).astype(np.float32)
        a, b = exp2_poly_fma_route(x_inf), exp2_poly_fma_route(x_big)
        assert np.array_equal(a, b)
        assert a[0] == -125.0 and a[1] == 0.0
