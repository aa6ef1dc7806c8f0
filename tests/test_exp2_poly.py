"""The FMA-pipe exponential used by the attention kernel, checked on the CPU against its error
bound: the coefficients hard-coded in the kernel are those the committed Remez derivation
produces, and a float32 model of the device steps stays within 2e-4 relative of 2^x."""
import os
import re

import numpy as np

from view_recon_b200.csrc import exp2_poly as ep

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_remez_error_bound():
    coef, err = ep.remez_exp2()
    assert err < 1e-4


def test_kernel_uses_the_derived_coefficients():
    text = open(os.path.join(ROOT, "view_recon_b200", "csrc", "sa_device.cuh")).read()
    body = text[text.index("float2 exp2_poly2"):]
    body = body[: body.index("\n}\n")]
    nums = [float(x) for x in re.findall(r"([0-9]\.[0-9]+e[-+][0-9]+)f", body)]
    coef, _ = ep.remez_exp2()
    # Horner order in the kernel: c3, c2, c1, c0
    want = [float(coef[3]), float(coef[2]), float(coef[1]), float(coef[0])]
    got = []
    for v in nums:
        if not got or got[-1] != v:
            got.append(v)
    assert np.allclose(got, want, rtol=1e-8, atol=0)


def test_emulated_device_routine_accuracy():
    coef, _ = ep.remez_exp2()
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float32),
                        np.array([0.0, -0.5, 0.5, -1e-7, 7.999], np.float32)])
    y = ep.emulate(x, coef).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 2e-4
    # clamp: far below the range the result is 2^-125, effectively zero for a softmax
    low = ep.emulate(np.array([-1e4, -np.inf], np.float32), coef).astype(np.float64)
    assert np.all(np.abs(low / 2.0 ** -125 - 1.0) < 2e-4)
