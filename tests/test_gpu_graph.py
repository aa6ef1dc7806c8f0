"""A layer call recorded as a CUDA graph replays to the same bits as the eager call.

Every step is one stream-ordered C call that allocates nothing, so
`SparseGlobalAttention.capture` records the whole call (pooling, scoring, selection -- a few
hundred launches in streamed mode -- and attention) and `replay()` re-runs it.  A replay must
give the eager call's bits on the captured inputs, and again after new inputs are written into
the same tensors (so the graph recomputes rather than repeats a result).
"""
import dataclasses

import pytest

from synth.workloads import VGGT_S16
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _eager(w, data):
    layer, _ = H.run_gpu(w, data)
    return layer


def _same(a, b):
    import torch
    assert torch.equal(a.buf.kept_cnt, b.buf.kept_cnt)
    assert torch.equal(a.buf.kept_idx, b.buf.kept_idx)
    assert torch.equal(a.buf.o, b.buf.o)
    assert torch.equal(a.buf.lse, b.buf.lse)


CASES = [
    VGGT_S16.scaled(heads=4),
    dataclasses.replace(VGGT_S16.scaled(heads=4), name="vggt_s16_streamed", streamed=True),
    # 384 frames: 4 224 tiles, two L2-sized blocks of score rows per head in streamed mode
    dataclasses.replace(VGGT_S16.scaled(heads=2), name="s384_streamed", frames=384, streamed=True),
]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_graph_replay_matches_eager(w):
    import torch
    from view_recon_b200 import sa
    from view_recon_b200.pipeline import SparseGlobalAttention
    first = H.inputs(w)
    second = H.inputs(w, seed=w.seed + 1)
    q, k, v = (H.to_device(first[x], w.dtype) for x in ("q", "k", "v"))
    layer = SparseGlobalAttention(w.heads, w.frames, w.tokens, w.k, w.tile, w.n_sink, w.dtype, w.landmark,
                                  w.streamed, w.head_dim)
    g = layer.capture(q, k, v)
    layer.buf.o.zero_()
    layer.buf.kept_cnt.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0
    _same(layer, _eager(w, first))

    # new inputs in the captured tensors: the replay recomputes every step
    for t, x in ((q, "q"), (k, "k"), (v, "v")):
        t.copy_(H.to_device(second[x], w.dtype))
    g.replay()
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0
    ref = _eager(w, second)
    assert not torch.equal(ref.buf.o, _eager(w, first).buf.o)
    _same(layer, ref)
    del g
