"""Per-head adaptive budgets (sa_head_budgets) against the oracle's head_budgets.

Bars: the per-head mean perplexity P_h within 1e-4 relative of the fp64 value (f32 scores and
exponentials over at most a few thousand candidates); the budget k_h equal to the oracle's,
except an off-by-one where beta * P_h lies within 1e-4 of a rounding boundary; the lists that
sa_select_topk_per_head then makes are the oracle's for those budgets up to near-tie swaps, and
the attention output follows the usual bar.
"""
import numpy as np
import pytest

import synth
from oracle import oracle as orc
from synth.workloads import VGGT_S16, Workload
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _pools(w, data):
    import torch
    from view_recon_b200 import sa
    q, k = H.to_device(data["q"], w.dtype), H.to_device(data["k"], w.dtype)
    shp = sa.shape_of(w)
    nt = sa.sa_num_tiles(shp)
    qp = torch.empty((w.heads, nt, 64), dtype=torch.float32, device="cuda")
    kp = torch.empty_like(qp)
    cnt = torch.empty((nt,), dtype=torch.int32, device="cuda")
    sk = torch.empty((w.heads, max(1, w.frames * w.n_sink), 64), dtype=q.dtype, device="cuda")
    sa.sa_tile_pool(shp, q, k, None, qp, kp, None, cnt, sk, None)
    return shp, qp, kp


def _budgets(shp, qp, kp, tau, beta, k_lo, k_hi):
    import torch
    from view_recon_b200 import sa
    bh = qp.shape[0]
    kh = torch.full((bh,), -1, dtype=torch.int32, device="cuda")
    perp = torch.zeros((bh,), dtype=torch.float32, device="cuda")
    ws = torch.empty((sa.sa_head_budget_workspace_size(shp),), dtype=torch.uint8, device="cuda")
    sa.sa_head_budgets(shp, qp, kp, tau, beta, k_lo, k_hi, kh, perp, ws)
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0
    return kh.cpu().numpy(), perp.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("tau,beta", [(16.0, 0.3), (64.0, 2.0), (4.0, 1.0)])
def test_head_budgets_match_oracle(tau, beta):
    w = VGGT_S16.scaled(heads=4)
    data = synth.generate(w)
    # heads with different spreads: scale the queries of two heads (a sharper / a flatter head)
    shp, qp, kp = _pools(w, data)
    qp[1] *= 3.0
    qp[2] *= 0.3
    kh, perp = _budgets(shp, qp, kp, tau, beta, 2, 150)
    g = H.geometry(w)
    qb = H.from_device(qp)
    kb = H.from_device(kp)
    p_ref, k_ref = orc.head_budgets(g, qb, kb, tau, beta, 2, 150)
    assert np.all(np.abs(perp - p_ref) <= 1e-4 * p_ref)
    for h in range(w.heads):
        assert orc.budget_matches(p_ref[h], beta, 2, 150, int(kh[h])), (h, kh[h], k_ref[h], p_ref[h])


def test_head_budgets_uniform_scores_are_dense():
    """Every key mean equal: each row's softmax is uniform, P_h is the candidate count and
    beta = 1 keeps every candidate."""
    import torch
    w = Workload("uniform", 6, 700, 3, 64, 128, 5, "bf16", 4, False, False, 64, 0, 0.7)
    data = synth.generate(w)
    shp, qp, kp = _pools(w, data)
    kp.copy_(kp[:, :1].expand_as(kp).contiguous())
    kh, perp = _budgets(shp, qp, kp, 16.0, 1.0, 0, 10_000)
    g = H.geometry(w)
    n_cand = len(orc.candidates(g, 0))
    assert np.all(np.abs(perp - n_cand) <= 1e-4 * n_cand)
    assert kh.tolist() == [n_cand] * w.heads
    torch.cuda.synchronize()


@pytest.mark.parametrize("streamed", [False, True])
def test_adaptive_layer_matches_oracle(streamed):
    """The layer call with adaptive budgets: budgets, per-head lists and attention output."""
    from view_recon_b200.pipeline import SparseGlobalAttention
    w = Workload("adaptive", 5, 900, 3, 64, 128, 5, "bf16", 30, False, streamed, 256, 0, 0.7)
    data = synth.generate(w)
    q, k, v = (H.to_device(data[x], w.dtype) for x in ("q", "k", "v"))
    ad = {"temperature": 24.0, "beta": 0.5, "k_lo": 1}
    layer = SparseGlobalAttention(w.heads, w.frames, w.tokens, w.k, streamed=streamed, adaptive=ad)
    layer.forward(q, k, v)
    import torch
    from view_recon_b200 import sa
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0
    g = H.geometry(w)
    Q, K, V = (orc.to_f64(data[x]) for x in ("q", "k", "v"))
    qb, kb, _, _, _, _ = orc.pool(g, Q, K, V)
    p_ref, _ = orc.head_budgets(g, qb, kb, 24.0, 0.5, 1, w.k)
    kh = H.from_device(layer.k_head)
    for h in range(w.heads):
        assert orc.budget_matches(p_ref[h], 0.5, 1, w.k, int(kh[h]))
    s = orc.scores(qb, kb)
    kept = H.kept_lists(layer)
    for h in range(w.heads):
        for i in range(g.nt):
            ok, msg = orc.selection_matches(g, s[h, i], i, int(kh[h]), kept[h][i])
            assert ok, "h=%d i=%d: %s" % (h, i, msg)
    O_ref, L_ref = orc.attend(g, Q, K, V, kept, 0.125)
    H.check_attention(H.from_device(layer.buf.o), H.from_device(layer.buf.lse), O_ref, L_ref)
