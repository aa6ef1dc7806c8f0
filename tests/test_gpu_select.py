"""Top-k selection alone, on score matrices built to stress it, against the oracle's rule.

The GPU selection receives f32 scores and the oracle ranks the very same f32 values (exactly
representable in fp64), so the kept lists must agree exactly, tie-breaking by lower index
included.  Rows are drawn from several families: Gaussian, integer-valued (many ties at the
threshold), constant (every candidate tied), a narrow band far from zero (ties after rounding,
one first-level bin), huge and tiny magnitudes, all negative, and two strided families: every 8th
tile (from tile 3) far above the rest, or far below it, which would mislead any selection that
estimated the threshold from a strided sample of the row.  Signed zeros are avoided: the
oracle treats -0 and +0 as equal, the kernel orders -0 below +0 (both are valid top-k sets).
Shapes cover the warp-per-row kernel (rows up to 2048 tiles; under 16 words of 32 tiles one tile per lane,
above one 32-tile word per lane) and the block-per-row kernel (longer rows), with and without
whole sink slots.
"""
import numpy as np
import pytest

from oracle import oracle as orc

pytestmark = pytest.mark.gpu


def score_rows(bh, nt, seed):
    """Row (h, i) belongs to family (i + 3h) mod 9."""
    rng = np.random.default_rng(seed)
    fam = (np.arange(nt)[None, :] + 3 * np.arange(bh)[:, None]) % 9          # [bh][nt]
    sampled = (np.arange(nt) % 8 == 3)[None, :]                               # every 8th tile from tile 3
    s = np.empty((bh, nt, nt), np.float32)
    for f in range(9):
        hs, is_ = np.nonzero(fam == f)
        n = rng.standard_normal((len(hs), nt))
        if f == 1:
            rows = rng.integers(-4, 5, (len(hs), nt)).astype(np.float64)        # many ties
        elif f == 2:
            rows = np.full((len(hs), nt), 1.25)                                 # all tied
        elif f == 3:
            rows = 100.0 + 1e-4 * n                                             # narrow band
        elif f == 4:
            rows = 1e30 * n                                                     # huge
        elif f == 5:
            rows = 1e-30 * n                                                    # tiny
        elif f == 6:
            rows = -np.abs(n) - 0.5                                             # all negative
        elif f == 7:
            rows = np.where(sampled, 10.0 + n, n)   # the strided tiles on top
        elif f == 8:
            rows = np.where(sampled, -10.0 + n, n)  # the strided tiles at the bottom
        else:
            rows = n                                                            # Gaussian
        s[hs, is_] = rows.astype(np.float32)
    s[s == 0] = np.float32(1e-20)  # no signed zeros
    return s


@pytest.mark.parametrize("frames,tokens,tile,n_sink,k,bh", [
    (40, 700, 128, 5, 17, 2),       # 240 tiles: warp-per-row kernel, one tile per lane
    (120, 1374, 128, 5, 130, 2),    # 1320 tiles: warp kernel, one 32-tile word per lane
    (100, 1374, 128, 256, 40, 1),   # 1100 tiles: the same with two whole sink slots per frame
    (7, 300, 64, 0, 3, 3),          # ragged frames, tile 64
    (5, 1374, 128, 0, 60, 1),       # k above the candidate count: every candidate kept
    (200, 1374, 128, 5, 130, 2),    # 2200 tiles: block-per-row kernel
    (190, 1374, 128, 256, 40, 1),   # block kernel, two whole sink slots per frame excluded
    (460, 1374, 128, 5, 327, 1),    # 5060 tiles, k = 327 (the 512/1024-frame budget)
    (30, 1374, 128, 256, 0, 1),     # k = 0: own frame only
    (40, 700, 128, 256, 9, 2),      # warp kernel with two whole sink slots per frame
])
def test_selection_exact_on_stress_rows(frames, tokens, tile, n_sink, k, bh):
    import torch
    from view_recon_b200 import sa
    g = orc.Geometry(frames, tokens, tile, n_sink)
    nt = g.nt
    s = score_rows(bh, nt, seed=frames * 1000 + nt)
    mk = orc.max_kept(g, k)
    kept_idx = torch.full((bh, nt, mk), -7, dtype=torch.int32, device="cuda")
    kept_cnt = torch.zeros((bh, nt), dtype=torch.int32, device="cuda")
    shp = sa.shape(bh, frames, tokens, 64, tile, n_sink, "bf16")
    sa.sa_select_topk(shp, torch.from_numpy(s).cuda(), None, None, k, kept_idx, kept_cnt, mk)
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0
    idx = kept_idx.cpu().numpy()
    cnt = kept_cnt.cpu().numpy()
    s64 = s.astype(np.float64)
    step = 1 if nt <= 1000 else 13  # long rows: every 13th row (still every family, 13 and 9 coprime)
    for h in range(bh):
        for i in range(0, nt, step):
            want = orc.select_row(g, s64[h, i], i, k)
            c = int(cnt[h, i])
            assert c == len(want), (h, i, c, len(want))
            assert idx[h, i, :c].tolist() == want.tolist(), (h, i, (i + 3 * h) % 9)
            assert (idx[h, i, c:] == -1).all()
