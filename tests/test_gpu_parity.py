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
    small("one_tile_per_frame", frames=6, tokens=100, k=2, landmark=True),
    # 130 special tokens: every frame's first key tile has no key row (own frame, listed first, so
    # a query tile's first item is masked whole) and its second starts at column 2
    small("sinks_fill_a_tile", frames=3, tokens=400, n_sink=130, k=2),
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


def test_host_pipeline_matches_device_calls():
    """Overlapped host-input calls give exactly the outputs of plain device calls."""
    import torch
    from view_recon_b200.pipeline import HostPipeline, SparseGlobalAttention
    w = small("hostpipe", frames=3, tokens=700, k=3)
    make = lambda: SparseGlobalAttention(w.heads, w.frames, w.tokens, w.k, w.tile, w.n_sink, w.dtype)
    pipe = HostPipeline(make)
    ref_layer = make()
    hosts, outs, refs = [], [], []
    for seed in (1, 2, 3, 4, 5):
        d = H.inputs(w, seed=seed)
        hq, hk, hv = (torch.from_numpy(d[x]).view(torch.bfloat16).pin_memory() for x in ("q", "k", "v"))
        ho = torch.empty_like(hq).pin_memory()
        hosts.append((hq, hk, hv))
        outs.append(ho)
        o, _ = ref_layer.forward(hq.cuda(), hk.cuda(), hv.cuda())
        refs.append(o.cpu())
    for (hq, hk, hv), ho in zip(hosts, outs):
        pipe.submit(hq, hk, hv, ho)
    pipe.synchronize()
    for ho, ref in zip(outs, refs):
        assert torch.equal(ho.view(torch.int16), ref.view(torch.int16))


@pytest.mark.parametrize("landmark,streamed", [(False, False), (True, False), (False, True)])
def test_per_head_budgets(landmark, streamed):
    """Per-head budgets (one head dense, one frame-only, two in between) through all four steps."""
    import torch
    from view_recon_b200 import sa
    from view_recon_b200.pipeline import SparseGlobalAttention
    w = small("per_head", frames=5, tokens=700, heads=4, k=3, landmark=landmark, streamed=streamed)
    g = H.geometry(w)
    budgets = [0, 2, 99, 7]
    data = H.inputs(w)
    q, k, v = (H.to_device(data[x], w.dtype) for x in ("q", "k", "v"))
    layer = SparseGlobalAttention(w.heads, w.frames, w.tokens, budgets, w.tile, w.n_sink, w.dtype, landmark,
                                  streamed)
    layer.forward(q, k, v)
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0
    Q, K, V = (orc.to_f64(data[x]) for x in ("q", "k", "v"))
    qb, kb, vb, cnt, _, _ = orc.pool(g, Q, K, V)
    s = orc.scores(qb, kb)
    kept = H.kept_lists(layer)
    assert H.from_device(layer.buf.kept_idx).shape[2] == orc.max_kept(g, max(budgets))
    ref = orc.select_per_head(g, s, budgets)
    for h, kh in enumerate(budgets):
        for i in range(g.nt):
            assert len(kept[h][i]) == len(ref[h][i])
            ok, msg = orc.selection_matches(g, s[h, i], i, kh, kept[h][i])
            assert ok, "h=%d i=%d: %s" % (h, i, msg)
    O_ref, L_ref = orc.attend(g, Q, K, V, kept, 0.125, landmark, kb, vb, cnt)
    H.check_attention(H.from_device(layer.buf.o), H.from_device(layer.buf.lse), O_ref, L_ref)


def test_per_head_budget_out_of_bound_is_reported_and_clamped():
    import torch
    from view_recon_b200 import sa
    w = small("per_head_bad", frames=3, tokens=300, heads=2, k=2, n_sink=0)
    g = H.geometry(w)
    layer, _ = H.run_gpu(w, H.inputs(w))
    torch.cuda.synchronize()
    bad = torch.tensor([1, 9], dtype=torch.int32, device="cuda")   # 9 > k_max = 2
    sa.sa_select_topk_per_head(layer.shape, layer.buf.scores, None, None, bad, 2, layer.buf.kept_idx,
                               layer.buf.kept_cnt, layer.max_kept)
    assert sa.sa_check_device_error() == sa.SA_ERR_INVALID_ARG
    cnt = H.from_device(layer.buf.kept_cnt)
    assert (cnt[0] == g.tpf + 1).all() and (cnt[1] == g.tpf + 2).all()
