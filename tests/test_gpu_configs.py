"""The five latent-point workloads at full size, in the launch configuration the benchmark times.

The 16-frame workload is compared in full (every head, every query tile).  The
128/512/1024-frame workloads run in full on the GPU; on two whole heads every
query tile's selection is compared with the oracle's fp64 score rows, and the
attention output on 64 seeded (head, query tile) items that always include the
first and last frame, a frame's sink-holding first tile and its partial last
tile.
"""
import numpy as np
import pytest

import synth
from oracle import oracle as orc
from synth.workloads import TINY, VGGT_S16, VGGT_S128, VGGT_S512, VGGT_S1024
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _sync_ok():
    import torch
    from view_recon_b200 import sa
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0


def test_tiny_workload_full():
    w = TINY
    data = synth.generate(w)
    layer, _ = H.run_gpu(w, data)
    _sync_ok()
    g = H.geometry(w)
    Q, K, V = (orc.to_f64(data[x]) for x in ("q", "k", "v"))
    qb, kb, vb, cnt, _, _ = orc.pool(g, Q, K, V)
    s = orc.scores(qb, kb)
    kept = H.kept_lists(layer)
    for h in range(w.heads):
        for i in range(g.nt):
            ok, msg = orc.selection_matches(g, s[h, i], i, w.k, kept[h][i])
            assert ok, msg
    O_ref, L_ref = orc.attend(g, Q, K, V, kept, 0.125)
    H.check_attention(H.from_device(layer.buf.o), H.from_device(layer.buf.lse), O_ref, L_ref)


def test_vggt16_workload_full():
    w = VGGT_S16
    data = synth.generate(w)
    layer, _ = H.run_gpu(w, data)
    _sync_ok()
    g = H.geometry(w)
    Q, K, V = (orc.to_f64(data[x]) for x in ("q", "k", "v"))
    qb, kb, vb, cnt, _, _ = orc.pool(g, Q, K, V)
    s = orc.scores(qb, kb)
    bound = 1e-5 * np.einsum("hid,hjd->hij", np.abs(qb), np.abs(kb)) + 1e-9
    assert np.all(np.abs(H.from_device(layer.buf.scores) - s) <= bound)
    kept = H.kept_lists(layer)
    swaps = 0
    for h in range(w.heads):
        for i in range(g.nt):
            ok, msg = orc.selection_matches(g, s[h, i], i, w.k, kept[h][i])
            assert ok, "h=%d i=%d: %s" % (h, i, msg)
            swaps += msg != "exact"
    O_ref, L_ref = orc.attend(g, Q, K, V, kept, 0.125)
    H.check_attention(H.from_device(layer.buf.o), H.from_device(layer.buf.lse), O_ref, L_ref)


def _sample_items(w, rng, n_random=26):
    """The first and last frame's sink-holding first tile and partial last tile, the same two
    tiles of a middle frame, and `n_random` seeded others."""
    tpf, nt = w.tpf, w.nt
    fixed = [0, tpf - 1, nt - tpf, nt - 1, (w.frames // 2) * tpf, (w.frames // 2) * tpf + tpf - 1]
    rest = np.setdiff1d(np.arange(nt), fixed)
    rand = rng.choice(rest, size=n_random, replace=False).tolist()
    return sorted(set(fixed + rand))


@pytest.mark.parametrize("w", [VGGT_S128, VGGT_S512, VGGT_S1024], ids=lambda w: w.name)
def test_large_workload_sampled(w):
    """Every query tile's selection of two whole heads (first and last) against the oracle's
    fp64 score rows, and the attention output of 32 (head, query tile) items per head (64 in
    all) recomputed by the oracle on the GPU's own lists."""
    import torch
    data = synth.generate(w)
    layer, (q, k, v) = H.run_gpu(w, data)
    _sync_ok()
    g = H.geometry(w)
    rng = np.random.default_rng(1234)
    heads = [0, w.heads - 1]
    kept_idx = H.from_device(layer.buf.kept_idx[heads])
    kept_cnt = H.from_device(layer.buf.kept_cnt)
    n_items = 0
    for hx, h in enumerate(heads):
        Qh, Kh, Vh = (orc.to_f64(data[x][h:h + 1]) for x in ("q", "k", "v"))
        qb, kb, vb, cnt, _, _ = orc.pool(g, Qh, Kh, Vh if w.landmark else None)
        gq = H.from_device(layer.buf.q_pool[h])
        gk = H.from_device(layer.buf.k_pool[h])
        assert np.all(np.abs(gq - qb[0]) <= 2e-5 + 1e-5 * np.abs(qb[0]))
        assert np.all(np.abs(gk - kb[0]) <= 2e-5 + 1e-5 * np.abs(kb[0]))
        s_all = orc.scores(qb, kb)[0]  # [nt][nt] fp64
        if not w.streamed:
            for i in _sample_items(w, rng, n_random=10):
                gs = H.from_device(layer.buf.scores[h, i])
                bound = 1e-5 * (np.abs(kb[0]) @ np.abs(qb[0, i])) + 1e-9
                assert np.all(np.abs(gs - s_all[i]) <= bound)
        lists = [kept_idx[hx, i, : kept_cnt[h, i]].astype(np.int64) for i in range(g.nt)]
        swaps = 0
        for i in range(g.nt):
            ok, msg = orc.selection_matches(g, s_all[i], i, w.k, lists[i])
            assert ok, "h=%d i=%d: %s" % (h, i, msg)
            swaps += msg != "exact"
        del s_all
        for i in _sample_items(w, rng):
            rows, (o_ref, l_ref) = orc.attend_tile(g, Qh, Kh, Vh, 0, i, lists[i], 0.125, w.landmark, kb, vb, cnt)
            o_gpu = H.from_device(layer.buf.o[h, torch.as_tensor(rows, device="cuda")])
            l_gpu = H.from_device(layer.buf.lse[h, torch.as_tensor(rows, device="cuda")])
            H.check_attention(o_gpu, l_gpu, o_ref, l_ref)
            n_items += 1
    assert n_items >= 64


def test_dense_control_sampled_rows_vggt16():
    import torch
    from view_recon_b200.pipeline import dense_attention
    w = VGGT_S16
    data = synth.generate(w, heads=2)
    q, k, v = (H.to_device(data[x], w.dtype) for x in ("q", "k", "v"))
    o, lse = dense_attention(q, k, v, w.frames, w.tokens, w.dtype)
    _sync_ok()
    rng = np.random.default_rng(7)
    rows = np.sort(rng.choice(w.L, size=256, replace=False))
    for h in range(2):
        Q, K, V = (orc.to_f64(data[x][h:h + 1]) for x in ("q", "k", "v"))
        O_ref, L_ref = orc.dense(Q[:, rows], K, V, 0.125)
        idx = torch.as_tensor(rows, device="cuda")
        H.check_attention(H.from_device(o[h, idx]), H.from_device(lse[h, idx]), O_ref[0], L_ref[0])
