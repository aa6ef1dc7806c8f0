"""Tile scores on the GPU against an fp64 product, element by element.

The bound is the fp32 accumulation bound used throughout: |gpu - fp64| <= 1e-5 * sum_e |q_e k_e| + 1e-9.
The kernel splits every f32 operand into two tf32 parts and sums three tf32 products, which stays
well inside it (about 2^-21 of sum_e |q_e k_e|).  Tile counts cover one and many 128-column chunks
per CTA and ragged edges: not a multiple of 64, of 128 or of 4 (scalar rather than 16-byte stores).
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bh,nt", [(2, 300), (1, 1100), (2, 1408), (3, 2050), (1, 1027)])
def test_scores_match_fp64(bh, nt):
    import torch
    from view_recon_b200 import sa
    rng = np.random.default_rng(nt)
    qp = (rng.standard_normal((bh, nt, 64)) / 11.3).astype(np.float32)
    kp = (rng.standard_normal((bh, nt, 64)) / 11.3).astype(np.float32)
    tokens = nt * 128  # one frame of nt tiles: only nt matters for this call
    shp = sa.shape(bh, 1, tokens, 64, 128, 0, "bf16")
    assert sa.sa_num_tiles(shp) == nt
    out = torch.full((bh, nt, nt), float("nan"), dtype=torch.float32, device="cuda")
    sa.sa_tile_scores(shp, torch.from_numpy(qp).cuda(), torch.from_numpy(kp).cuda(), out)
    torch.cuda.synchronize()
    got = out.cpu().numpy().astype(np.float64)
    q64, k64 = qp.astype(np.float64), kp.astype(np.float64)
    ref = np.einsum("hid,hjd->hij", q64, k64)
    bound = 1e-5 * np.einsum("hid,hjd->hij", np.abs(q64), np.abs(k64)) + 1e-9
    assert np.isfinite(got).all()
    assert (np.abs(got - ref) <= bound).all()
