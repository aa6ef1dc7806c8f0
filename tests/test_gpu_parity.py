"""GPU vs fp64 oracle, step by step, on small shapes that span several tiles and ragged tails.

Bars:
  pooling      |gpu - oracle| <= 2e-5 + 1e-5 |oracle|  (f32 sums of <= 128 rows), sinks and counts exact
  scores       |gpu - oracle| <= 1e-5 * sum_e |q_e k_e| + 1e-9  (f32 dot products of f32 means)
  selection    oracle's kept set, up to swaps of near-equal fp64 scores (1e-4 relative)
  attention    oracle recomputed on the GPU's own lists: max-abs <= 2e-2, mean-abs <= 2e-3,
               LSE abs <= 1e-2
"""
import numpy as np
import pytest

from oracle import oracle as orc
from synth.workloads import TINY, VGGT_S16, Workload
from tests import helpers as H

pytestmark = pytest.mark.gpu


def small(name, frames=3, tokens=1374, heads=2, tile=128, n_sink=5, dtype="bf16", k=4, landmark=False,
          streamed=False, n_points=256, window=0, p_assign=0.7):
    return Workload(name, frames, tokens, heads, 64, tile, n_sink, dtype, k, landmark, streamed, n_points,
                    window, p_assign)


CASES = [
    TINY,
    small("vggt3_k4"),
    small("vggt3_k4_landmark", landmark=True),
    small("ragged300_nosink", tokens=300, n_sink=0, frames=4, k=3),
    small("k0_frame_attention", k=0),
    small("k_all_is_dense", frames=2, tokens=400, k=1000),
    small("one_frame", frames=1, tokens=700, k=3),
    small("bf16_tile64", tile=64, frames=2, tokens=300, k=5),
    small("f32_tile128", dtype="f32", frames=2, tokens=300, k=2),
    small("streamed_select", frames=4, tokens=600, k=3, streamed=True),
    small("window_landmark_streamed", frames=6, tokens=500, k=4, landmark=True, streamed=True, window=2),
]


def _run_case(w, data):
    layer, _ = H.run_gpu(w, data)
    import torch
    torch.cuda.synchronize()
    from view_recon_b200 import sa
    assert sa.sa_check_device_error() == 0
    return layer


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_every_step_matches_oracle(w):
    data = H.inputs(w)
    layer = _run_case(w, data)
    g = H.geometry(w)
    Q, K, V = (orc.to_f64(data[x]) for x in ("q", "k", "v"))
    qb, kb, vb, cnt, sk, sv = orc.pool(g, Q, K, V)

    # step 1: pooling
    b = layer.buf
    for got, ref in ((b.q_pool, qb), (b.k_pool, kb)):
        gv = H.from_device(got)
        assert np.all(np.abs(gv - ref) <= 2e-5 + 1e-5 * np.abs(ref))
    if w.landmark:
        gv = H.from_device(b.v_pool)
        assert np.all(np.abs(gv - vb) <= 2e-5 + 1e-5 * np.abs(vb))
    assert np.array_equal(H.from_device(b.k_cnt), cnt)
    if w.n_sink:
        assert np.array_equal(H.from_device(b.sink_k)[:, : w.frames * w.n_sink], sk)
        assert np.array_equal(H.from_device(b.sink_v)[:, : w.frames * w.n_sink], sv)

    # step 2: scores (materialised mode)
    s = orc.scores(qb, kb)
    if not w.streamed:
        bound = 1e-5 * np.einsum("hid,hjd->hij", np.abs(qb), np.abs(kb)) + 1e-9
        assert np.all(np.abs(H.from_device(b.scores) - s) <= bound)

    # step 3: selection
    kept = H.kept_lists(layer)
    idx = H.from_device(b.kept_idx)
    assert idx.shape[2] == orc.max_kept(g, w.k)
    for h in range(w.heads):
        for i in range(g.nt):
            ok, msg = orc.selection_matches(g, s[h, i], i, w.k, kept[h][i])
            assert ok, "h=%d i=%d: %s" % (h, i, msg)
            assert np.all(idx[h, i, len(kept[h][i]):] == -1)

    # step 4: attention on the GPU's own lists
    O_ref, L_ref = orc.attend(g, Q, K, V, kept, 1.0 / np.sqrt(w.head_dim), w.landmark, kb, vb, cnt)
    H.check_attention(H.from_device(b.o), H.from_device(b.lse), O_ref, L_ref)


@pytest.mark.parametrize("w", [TINY, small("dense_bf16", frames=3, tokens=700),
                               small("dense_f32_t128", dtype="f32", frames=2, tokens=300)],
                         ids=lambda w: w.name)
def test_dense_control_matches_textbook(w):
    from view_recon_b200.pipeline import dense_attention
    data = H.inputs(w)
    q, k, v = (H.to_device(data[x], w.dtype) for x in ("q", "k", "v"))
    o, lse = dense_attention(q, k, v, w.frames, w.tokens, w.dtype)
    Q, K, V = (orc.to_f64(data[x]) for x in ("q", "k", "v"))
    O_ref, L_ref = orc.dense(Q, K, V, 1.0 / np.sqrt(w.head_dim))
    H.check_attention(H.from_device(o), H.from_device(lse), O_ref, L_ref)


def test_all_tiles_kept_equals_dense_on_gpu():
    # k >= candidates and sinks attended once: the sparse call computes dense attention
    w = small("k_all", frames=2, tokens=400, k=10 ** 6, n_sink=5)
    from view_recon_b200.pipeline import dense_attention
    data = H.inputs(w)
    layer, (q, k, v) = H.run_gpu(w, data)
    o_d, l_d = dense_attention(q, k, v, w.frames, w.tokens, w.dtype)
    H.check_attention(H.from_device(layer.buf.o), H.from_device(layer.buf.lse), H.from_device(o_d),
                      H.from_device(l_d), max_abs=2e-2, mean_abs=2e-3)


def test_equal_scores_pick_lowest_indices():
    # every key row identical -> every tile mean identical -> every score in a row ties
    w = small("ties", frames=4, tokens=256, k=3, n_sink=0)
    data = H.inputs(w)
    data["k"][:] = data["k"][:, :1, :]
    layer, _ = H.run_gpu(w, data)
    kept = H.kept_lists(layer)
    g = H.geometry(w)
    for h in range(w.heads):
        for i in range(g.nt):
            cand = orc.candidates(g, i)
            want = np.sort(np.concatenate([g.own_frame_tiles(i), cand[:3]]))
            assert kept[h][i].tolist() == want.tolist()


def test_out_of_range_list_entry_is_reported_not_faulted():
    import torch
    from view_recon_b200 import sa
    w = small("badlist", frames=2, tokens=300, k=1, n_sink=0)
    data = H.inputs(w)
    layer, (q, k, v) = H.run_gpu(w, data)
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0
    layer.buf.kept_idx[0, 0, 0] = layer.nt + 7     # planted bad entry, host side
    layer.attend(q, k, v)
    assert sa.sa_check_device_error() == sa.SA_ERR_BAD_LIST
    assert sa.sa_check_device_error() == 0         # the word is cleared by the read


def test_argument_errors_touch_nothing():
    import torch
    from view_recon_b200 import sa
    w = small("args", frames=2, tokens=300, k=1, n_sink=0)
    data = H.inputs(w)
    layer, (q, k, v) = H.run_gpu(w, data)
    before = layer.buf.o.clone()
    shp = sa.shape(w.heads, w.frames, w.tokens, 64, 128, 0, "bf16")
    with pytest.raises(sa.SaError) as e:
        sa.sa_sparse_attn_fwd(shp, q, k, v, layer.buf.kept_idx, layer.buf.kept_cnt, 0, None, None, False,
                              None, None, None, None, layer.buf.o)
    assert e.value.status == sa.SA_ERR_INVALID_ARG
    bad = sa.shape(w.heads, w.frames, w.tokens, 32, 128, 0, "bf16")
    with pytest.raises(sa.SaError) as e:
        sa.sa_dense_attn_fwd(bad, q, k, v, None, layer.buf.o)
    assert e.value.status == sa.SA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.equal(before, layer.buf.o)
