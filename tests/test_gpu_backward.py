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


def _rows_of(t, h, rows):
    import torch
    return H.from_device(t[h, torch.as_tensor(np.asarray(rows), device=t.device)])


@pytest.mark.parametrize("wname", ["vggt_s128_n1374", "vggt_s512_n1374_landmark"])
def test_backward_large_workload_sampled(wname):
    """The benchmark's layer call at 128 frames (k = 130) and 512 frames (landmarks), forward and
    backward over all 16 heads; compared on samples the oracle can finish in seconds: dq of
    seeded query tiles of the first and last head (first and last frame, a frame's sink tile and
    partial tile among them), and at 128 frames dk, dv of one key tile per head, whose rows the
    oracle completes by running every query tile that lists it.  (A key tile's landmark gradient at
    512 frames gathers from nearly every query tile, beyond a sampled check.)"""
    import torch
    from synth.workloads import BY_NAME
    from view_recon_b200 import sa
    w = BY_NAME[wname]
    data = H.inputs(w)
    layer, (q, k, v) = H.run_gpu(w, data)
    do_h = bf16_normal((w.heads, w.L, 64), 13)
    d_o = H.to_device(do_h, "bf16")
    dq, dk, dv = layer.backward(q, k, v, d_o)
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0
    g = H.geometry(w)
    tpf, nt = w.tpf, g.nt
    rng = np.random.default_rng(21)
    tiles = sorted(set([0, tpf - 1, nt - tpf, nt - 1, (w.frames // 2) * tpf + 3] +
                       rng.choice(nt, size=3, replace=False).tolist()))
    for h in (0, w.heads - 1):
        Qh, Kh, Vh = (orc.to_f64(data[x][h:h + 1]) for x in ("q", "k", "v"))
        dOh = orc.to_f64(do_h[h:h + 1])
        idx = H.from_device(layer.buf.kept_idx[h]).astype(np.int64)
        cnt = H.from_device(layer.buf.kept_cnt[h]).astype(np.int64)
        kept = [idx[i, :cnt[i]] for i in range(nt)]
        ref_q, _, _ = orc.attend_backward(g, Qh, Kh, Vh, [kept], dOh, 0.125, w.landmark,
                                          items=[(0, i) for i in tiles])
        rows = np.concatenate([g.tile_rows(i) for i in tiles])
        check_grad("dq h=%d" % h, _rows_of(dq, h, rows), ref_q[0, rows])
        if w.landmark:
            continue
        # one key tile per head: an interior tile of a random frame, then a frame's sink-holding tile
        j_pick = int(rng.integers(1, tpf)) + tpf * int(rng.integers(0, w.frames)) if h == 0 else 2 * tpf
        for j in (j_pick,):
            users = [i for i in range(nt) if j in set(kept[i].tolist())]
            _, ref_k, ref_v = orc.attend_backward(g, Qh, Kh, Vh, [kept], dOh, 0.125, False,
                                                  items=[(0, i) for i in users])
            kr = g.tile_key_rows(j)  # non-sink rows: complete with these query tiles
            check_grad("dk h=%d j=%d" % (h, j), _rows_of(dk, h, kr), ref_k[0, kr])
            check_grad("dv h=%d j=%d" % (h, j), _rows_of(dv, h, kr), ref_v[0, kr])


@pytest.mark.parametrize("landmark", [False, True])
def test_backward_per_head_budgets(landmark):
    """Per-head budgets (k = 0, 3, 9): rows of the smaller budgets hold fewer tiles than max_kept,
    the rest of each row being -1; every gradient of every head against the oracle."""
    import torch
    from view_recon_b200 import sa
    from view_recon_b200.pipeline import SparseGlobalAttention
    w = Workload("per_head", 5, 300, 3, 64, 128, 5, "bf16", 9, landmark, False, 256, 0, 0.7)
    data = H.inputs(w)
    q, k, v = (H.to_device(data[x], "bf16") for x in ("q", "k", "v"))
    layer = SparseGlobalAttention(w.heads, w.frames, w.tokens, [0, 3, 9], landmark=landmark)
    layer.forward(q, k, v)
    do_h = bf16_normal((w.heads, w.L, 64), 17)
    dq, dk, dv = layer.backward(q, k, v, H.to_device(do_h, "bf16"))
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0
    cnt = H.from_device(layer.buf.kept_cnt)
    assert cnt[0].max() < layer.max_kept == cnt[2].max()  # short rows are present
    compare(w, layer, data, do_h, (H.from_device(dq), H.from_device(dk), H.from_device(dv)), range(w.heads))
