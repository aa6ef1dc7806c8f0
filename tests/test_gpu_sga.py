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
