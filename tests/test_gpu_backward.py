"""Backward of the block-sparse attention on the GPU against the fp64 oracle.

The oracle differentiates the same layer call (the GPU's own kept lists held fixed).  Bars,
per head and per gradient tensor, derived from the kernel's arithmetic (bf16 operands, P and dS
rounded to bf16 before their products, f32 accumulation, bf16 outputs), whose emulation on a
VGGT-like head gives max errors near 0.5 % of max|ref| and mean errors near 0.3 % of mean|ref|:
    max|gpu - ref| <= 2e-2 * max|ref|   and   mean|gpu - ref| <= 1e-2 * mean|ref|.
Cases: ragged frames (partial last tile), sinks or none, landmarks, every tile listed (the
dense gradients), key tiles attended by more query tiles than one dK/dV unit holds (their
contributions meet in the fp32 accumulators), the VGGT frame, and the benchmark's 16-frame
layer call in full on two heads.
"""
import numpy as np
import pytest

from oracle import oracle as orc
from synth.workloads import VGGT_S16, Workload
from tests import helpers as H

pytestmark = pytest.mark.gpu


def check_grad(name, got, ref, max_rel=2e-2, mean_rel=1e-2):
    assert np.isfinite(got).all(), "%s: non-finite gradient" % name
    err = np.abs(got - ref)
    scale_max, scale_mean = np.abs(ref).max(), np.abs(ref).mean()
    assert err.max() <= max_rel * scale_max, "%s: max err %.3g > %.3g" % (name, err.max(), max_rel * scale_max)
    assert err.mean() <= mean_rel * scale_mean, "%s: mean err %.3g > %.3g" % (name, err.mean(), mean_rel * scale_mean)


def bf16_normal(shape, seed):
    f = np.random.default_rng(seed).standard_normal(shape).astype(np.float32)
    b = f.view(np.uint32)
    return ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)


def run_case(w, seed=5):
    import torch
    from view_recon_b200 import sa
    data = H.inputs(w)
    layer, (q, k, v) = H.run_gpu(w, data)
    do_h = bf16_normal((w.heads, w.L, 64), seed)
    d_o = H.to_device(do_h, "bf16")
    dq, dk, dv = layer.backward(q, k, v, d_o)
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0
    return layer, data, do_h, (H.from_device(dq), H.from_device(dk), H.from_device(dv))


def compare(w, layer, data, do_h, got, heads):
    g = H.geometry(w)
    kept = H.kept_lists(layer)
    for h in heads:
        Q, K, V = (orc.to_f64(data[x][h:h + 1]) for x in ("q", "k", "v"))
        dO = orc.to_f64(do_h[h:h + 1])
        ref = orc.attend_backward(g, Q, K, V, [kept[h]], dO, 0.125, w.landmark)
        for name, a, b in zip(("dq", "dk", "dv"), got, ref):
            check_grad("%s h=%d" % (name, h), a[h], b[0])
    return kept


CASES = [
    # name, frames, tokens, heads, k, n_sink, landmark
    ("ragged_sinks", 3, 300, 2, 2, 5, False),
    ("ragged_sinks_landmark", 3, 300, 2, 2, 5, True),
    ("exact_tiles_no_sinks", 4, 256, 2, 1, 0, False),
    ("vggt_frame", 6, 1374, 2, 8, 5, False),
    ("vggt_frame_landmark", 6, 1374, 2, 8, 5, True),
    ("long_reverse_lists", 40, 256, 1, 70, 5, False),
    ("long_reverse_lists_landmark", 40, 256, 1, 20, 5, True),
]


@pytest.mark.parametrize("name,frames,tokens,heads,k,n_sink,landmark", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_oracle(name, frames, tokens, heads, k, n_sink, landmark):
    w = Workload(name, frames, tokens, heads, 64, 128, n_sink, "bf16", k, landmark, False, 256, 0, 0.7)
    layer, data, do_h, got = run_case(w)
    compare(w, layer, data, do_h, got, range(heads))


def test_backward_all_tiles_is_dense():
    w = Workload("all_tiles", 3, 300, 1, 64, 128, 5, "bf16", 99, False, False, 256, 0, 0.7)
    layer, data, do_h, got = run_case(w)
    kept = compare(w, layer, data, do_h, got, [0])
    g = H.geometry(w)
    assert all(len(x) == g.nt for x in kept[0])
    Q, K, V = (orc.to_f64(data[x]) for x in ("q", "k", "v"))
    ref = orc.dense_backward(Q, K, V, orc.to_f64(do_h), 0.125)
    for name, a, b in zip(("dq", "dk", "dv"), got, ref):
        check_grad(name, a, b)


def test_backward_vggt16_full_call_two_heads():
    """The benchmark's layer call (16 frames x 1374 tokens, 16 heads, k = 35) forward and
    backward on the GPU; every gradient of the first and last head against the oracle."""
    w = VGGT_S16
    layer, data, do_h, got = run_case(w, seed=11)
    compare(w, layer, data, do_h, got, [0, w.heads - 1])
