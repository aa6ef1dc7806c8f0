"""Derive the cubic used for 2^f, f in [-1/2, 1/2], by the FMA-pipe exponential in k_attn_tc.cuh.

Method: Remez exchange on the relative error of a degree-3 polynomial against 2^f,
started from the Chebyshev extrema.  2^x is then reconstructed as p(x - n) * 2^n with
n = round(x) obtained by the classic magic-number rounding (adding 1.5 * 2^23 in float32)
and 2^n applied by adding n to the exponent field.  Run as a script to print the
float32 coefficients that the kernel hard-codes.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3


def remez_exp2(degree: int = DEGREE, iters: int = 40):
    f = np.linspace(-0.5, 0.5, 400001)
    pts = 0.5 * np.cos(np.pi * np.arange(degree + 2) / (degree + 1))[::-1]
    coef = None
    for _ in range(iters):
        A = np.zeros((degree + 2, degree + 2))
        for i, p in enumerate(pts):
            A[i, : degree + 1] = p ** np.arange(degree + 1)
            A[i, degree + 1] = (-1) ** i * 2.0 ** p
        sol = np.linalg.solve(A, 2.0 ** pts)
        coef = sol[: degree + 1]
        err = np.polyval(coef[::-1], f) / 2.0 ** f - 1.0
        idx = np.where(np.diff(np.sign(np.diff(err))) != 0)[0] + 1
        ext = np.concatenate([[0], idx, [len(f) - 1]])
        if len(ext) != degree + 2:
            break
        pts = f[ext]
    err = np.polyval(coef[::-1], f) / 2.0 ** f - 1.0
    return coef.astype(np.float32), float(np.abs(err).max())


def emulate(x: np.ndarray, coef: np.ndarray) -> np.ndarray:
    """float32 model of the device routine (clamp, magic rounding, Horner, exponent add)."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    fr = (x - n).astype(np.float32)
    p = np.float32(coef[3])
    for c in (coef[2], coef[1], coef[0]):
        p = (p * fr + np.float32(c)).astype(np.float32)
    bits = p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << np.uint64(23))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    c, e = remez_exp2()
    print("max relative error on [-1/2, 1/2]: %.3e" % e)
    for i, v in enumerate(c):
        print("c%d = %.9ef" % (i, v))
