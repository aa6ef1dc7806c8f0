"""The split-precision dot product behind the tile scores, emulated on the CPU.

The score kernel splits every f32 operand x into hi = rn_tf32(x) and lo = rn_tf32(x - hi) (tf32: 10
stored mantissa bits, round to nearest with ties away from zero, as `cvt.rna.tf32.f32`), and takes
a . b as lo.hi + hi.lo + hi.hi.  Each tf32 product is exact in f32 (11 x 11 significant bits), so
the only errors are the representation error of the split (|x - hi - lo| <= 2^-22 |x|), the dropped
lo.lo term (<= 2^-22 |a||b|) and the f32 accumulation.  These tests emulate the split exactly and
check the bound the header states, |s - a.b| <= 2^-21 sum_e |a_e b_e| (plus the f32 accumulation
of 192 terms), against fp64 on random and adversarial inputs.  They pin the method, not the kernel
(the GPU tests compare the kernel with fp64 under the looser 1e-5 bound).
"""
import numpy as np


def tf32_rna(x: np.ndarray) -> np.ndarray:
    """f32 -> nearest tf32 (10 stored mantissa bits), ties away from zero; kept as f32."""
    b = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x1000) & 0xFFFFE000  # add half of the dropped 13 bits, then truncate
    return b.astype(np.uint32).view(np.float32)


def split(x):
    hi = tf32_rna(x)
    lo = tf32_rna((np.asarray(x, np.float32) - hi).astype(np.float32))
    return hi, lo


def split_dot(a, b):
    """lo.hi + hi.lo + hi.hi with exact products and an f32 running sum (the tensor cores sum in
    another order; the bound below holds for any order of 192 f32 additions)."""
    ah, al = split(a)
    bh, bl = split(b)
    acc = np.zeros(a.shape[:-1], np.float32)
    for e in range(a.shape[-1]):
        for x, y in ((al, bh), (ah, bl), (ah, bh)):
            p = (x[..., e].astype(np.float64) * y[..., e].astype(np.float64)).astype(np.float32)
            acc = (acc + p).astype(np.float32)
    return acc


def check(a, b):
    got = split_dot(a, b).astype(np.float64)
    a64, b64 = a.astype(np.float64), b.astype(np.float64)
    ref = (a64 * b64).sum(-1)
    mag = np.abs(a64 * b64).sum(-1)
    # 2^-21 for the split and lo.lo, plus f32 rounding of 192 partial sums (each <= 2^-24 of mag)
    bound = (2.0 ** -21 + 192 * 2.0 ** -24) * mag + 1e-45
    assert (np.abs(got - ref) <= bound).all()
    return float((np.abs(got - ref) / np.maximum(mag, 1e-300)).max())


def test_split_is_exact_to_22_bits():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(100000) * 10.0 ** rng.uniform(-20, 20, 100000)).astype(np.float32)
    hi, lo = split(x)
    r = np.abs(x.astype(np.float64) - hi.astype(np.float64) - lo.astype(np.float64))
    assert (r <= 2.0 ** -22 * np.abs(x.astype(np.float64))).all()
    # hi keeps 10 mantissa bits, lo as well
    assert ((hi.view(np.uint32) & 0x1FFF) == 0).all() and ((lo.view(np.uint32) & 0x1FFF) == 0).all()


def test_tf32_rounding_matches_its_definition():
    # ties go away from zero; just above / below a tie round to the nearer neighbour
    one = np.float32(1.0)
    ulp = np.float32(2.0 ** -10)
    tie = np.float32(1.0 + 2.0 ** -11)
    assert tf32_rna(np.array([tie], np.float32))[0] == one + ulp
    assert tf32_rna(np.array([-tie], np.float32))[0] == -(one + ulp)
    below = np.nextafter(tie, np.float32(0))
    assert tf32_rna(np.array([below], np.float32))[0] == one


def test_pooled_scores_within_bound():
    rng = np.random.default_rng(7)
    a = (rng.standard_normal((512, 64)) / 11.3).astype(np.float32)   # tile means of unit-variance rows
    b = (rng.standard_normal((512, 64)) / 11.3).astype(np.float32)
    worst = check(a, b)
    assert worst < 2.0 ** -20


def test_cancellation_and_wide_ranges_within_bound():
    rng = np.random.default_rng(11)
    a = rng.standard_normal((256, 64)).astype(np.float32)
    b = a.copy()
    b[:, 32:] = -b[:, :32]          # a.b cancels to about zero: the bound is relative to sum |a_e b_e|
    a[:, 32:] = a[:, :32]
    check(a, b)
    c = (rng.standard_normal((256, 64)) * 10.0 ** rng.uniform(-15, 15, (256, 64))).astype(np.float32)
    d = (rng.standard_normal((256, 64)) * 10.0 ** rng.uniform(-15, 15, (256, 64))).astype(np.float32)
    check(c, d)


def test_single_tf32_product_would_not_do():
    """The reason for the split: one tf32 product misses the 1e-6-relative accuracy that a 1e-4
    swap rule on near-tied scores needs by orders of magnitude."""
    rng = np.random.default_rng(3)
    a = (rng.standard_normal((512, 64)) / 11.3).astype(np.float32)
    b = (rng.standard_normal((512, 64)) / 11.3).astype(np.float32)
    one = (tf32_rna(a).astype(np.float64) * tf32_rna(b).astype(np.float64)).sum(-1)
    ref = (a.astype(np.float64) * b.astype(np.float64)).sum(-1)
    mag = np.abs(a.astype(np.float64) * b.astype(np.float64)).sum(-1)
    assert (np.abs(one - ref) / mag).max() > 1e-4
