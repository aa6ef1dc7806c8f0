"""Subsampled global attention (AVGGT SGA) on the GPU against the fp64 oracle.

Bars as for the sparse layer: max-abs <= 2e-2 and mean-abs <= 2e-3 on O, LSE abs <= 1e-2.
Shapes: the VGGT frame (5 special tokens + a 37 x 37 grid) at strides 3 and 9, a ragged grid
whose windows do not divide it, no special tokens, stride 1 (no discarded tokens: dense).
"""
import numpy as np
import pytest

from oracle import oracle as orc
from synth.workloads import Workload
from tests import helpers as H

pytestmark = pytest.mark.gpu


def bf16_inputs(heads, L, seed):
    """Seeded N(0, 1) inputs rounded to bf16 bit patterns (round to nearest even)."""
    rng = np.random.default_rng(seed)
    out = {}
    for name in ("q", "k", "v"):
        f = rng.standard_normal((heads, L, 64)).astype(np.float32)
        b = f.view(np.uint32)
        out[name] = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)
    return out


CASES = [
    # frames, n_special, grid_h, grid_w, s_h, s_w, source
    (3, 5, 37, 37, 3, 3, "synth"),
    (2, 5, 37, 37, 9, 9, "synth"),
    (2, 2, 10, 12, 3, 5, "normal"),
    (4, 0, 13, 11, 4, 5, "normal"),
    (2, 3, 6, 7, 1, 1, "normal"),
]


@pytest.mark.parametrize("frames,ns,gh,gw,sh,sw,src", CASES)
def test_sga_matches_oracle(frames, ns, gh, gw, sh, sw, src):
    import torch
    from view_recon_b200 import sa
    from view_recon_b200.pipeline import SubsampledGlobalAttention
    heads, N = 2, ns + gh * gw
    L = frames * N
    if src == "synth":
        w = Workload("sga", frames, N, heads, 64, 128, ns, "bf16", 0, False, False, 256, 0, 0.7)
        data = H.inputs(w)
    else:
        data = bf16_inputs(heads, L, seed=frames * 100 + gh)
    q, k, v = (H.to_device(data[x], "bf16") for x in ("q", "k", "v"))
    layer = SubsampledGlobalAttention(heads, frames, N, grid=(gh, gw), stride=(sh, sw), n_special=ns)
    layer.forward(q, k, v)
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0
    Q, K, V = (orc.to_f64(data[x]) for x in ("q", "k", "v"))
    O_ref, L_ref = orc.sga(Q, K, V, frames, N, ns, gh, gw, sh, sw, 0.125)
    H.check_attention(H.from_device(layer.o), H.from_device(layer.lse), O_ref, L_ref)
    if sh == 1 and sw == 1:
        O_d, L_d = orc.dense(Q, K, V, 0.125)
        H.check_attention(H.from_device(layer.o), H.from_device(layer.lse), O_d, L_d)


def _sga_rows(w, rng, stride, n_random=48):
    """Query rows that reach every case of the layer: special tokens, kept and discarded
    patches, the last patch of a frame, in the first, middle and last frame, plus random rows."""
    g = int(round((w.tokens - w.n_sink) ** 0.5))
    fixed = []
    for f in (0, w.frames // 2, w.frames - 1):
        base = f * w.tokens
        fixed += [base, base + w.n_sink - 1,                       # special tokens
                  base + w.n_sink,                                 # patch (0, 0): kept
                  base + w.n_sink + 1,                             # patch (0, 1): discarded
                  base + w.n_sink + stride * g + stride,           # kept, interior
                  base + w.tokens - 1]                             # last patch of the frame
    rand = rng.choice(w.L, size=n_random, replace=False).tolist()
    return sorted(set(fixed + rand))


@pytest.mark.parametrize("wname,stride", [("vggt_s16_n1374", 3), ("vggt_s16_n1374", 9),
                                          ("vggt_s128_n1374", 3)])
def test_sga_full_size_sampled_rows(wname, stride):
    """The benchmark's SGA launch (every head of the workload, 37 x 37 patch grid) compared with
    the oracle on sampled query rows of the first and last head."""
    import torch
    import synth
    from view_recon_b200 import sa
    from view_recon_b200.pipeline import SubsampledGlobalAttention
    from synth.workloads import VGGT_S16, VGGT_S128
    w = {"vggt_s16_n1374": VGGT_S16, "vggt_s128_n1374": VGGT_S128}[wname]
    grid = int(round((w.tokens - w.n_sink) ** 0.5))
    data = synth.generate(w)
    q, k, v = (H.to_device(data[x], w.dtype) for x in ("q", "k", "v"))
    layer = SubsampledGlobalAttention(w.heads, w.frames, w.tokens, (grid, grid), (stride, stride),
                                      w.n_sink, w.dtype, w.head_dim)
    layer.forward(q, k, v)
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0
    rng = np.random.default_rng(stride * 1000 + w.frames)
    rows = _sga_rows(w, rng, stride)
    idx = torch.as_tensor(rows, device="cuda")
    for h in (0, w.heads - 1):
        Q, K, V = (orc.to_f64(data[x][h:h + 1]) for x in ("q", "k", "v"))
        O_ref, L_ref = orc.sga(Q, K, V, w.frames, w.tokens, w.n_sink, grid, grid, stride, stride,
                               0.125, rows=rows)
        H.check_attention(H.from_device(layer.o[h, idx]), H.from_device(layer.lse[h, idx]),
                          O_ref[0, rows], L_ref[0, rows])
