"""A head shard of one layer call computes exactly its part of that call.

`bench.py --shard heads` splits one layer call over GPUs by heads: rank r draws heads
[r*H/N, (r+1)*H/N) of the seeded draw (the generator's head offset) and runs the four steps on
them alone.  Heads are independent problems end to end, so a shard must give, on its heads,
the oracle's result for those heads of the full draw, and the very same bits as the full
16-head call on the same GPU.
"""
import numpy as np
import pytest

import synth
from oracle import oracle as orc
from synth.workloads import VGGT_S16
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world,rank", [(4, 2), (8, 7)])
def test_head_shard_is_its_slice_of_the_full_call(world, rank):
    import torch
    from view_recon_b200 import sa
    w = VGGT_S16
    hl = w.heads // world
    h0 = rank * hl
    full = synth.generate(w)
    part = synth.generate(w.scaled(heads=hl), head0=h0)
    for x in ("q", "k", "v"):
        assert np.array_equal(part[x], full[x][h0:h0 + hl])

    shard, _ = H.run_gpu(w.scaled(heads=hl), part)
    whole, _ = H.run_gpu(w, full)
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0

    # the same bits as the full call on these heads
    sl = slice(h0, h0 + hl)
    assert torch.equal(shard.buf.kept_cnt, whole.buf.kept_cnt[sl])
    assert torch.equal(shard.buf.kept_idx, whole.buf.kept_idx[sl])
    assert torch.equal(shard.buf.o, whole.buf.o[sl])
    assert torch.equal(shard.buf.lse, whole.buf.lse[sl])

    # the oracle on the same heads of the full draw
    g = H.geometry(w)
    Q, K, V = (orc.to_f64(full[x][sl]) for x in ("q", "k", "v"))
    qb, kb, _, _, _, _ = orc.pool(g, Q, K, V)
    s = orc.scores(qb, kb)
    kept = H.kept_lists(shard)
    for h in range(hl):
        for i in range(g.nt):
            ok, msg = orc.selection_matches(g, s[h, i], i, w.k, kept[h][i])
            assert ok, "head %d tile %d: %s" % (h0 + h, i, msg)
    O_ref, L_ref = orc.attend(g, Q, K, V, kept, 0.125)
    H.check_attention(H.from_device(shard.buf.o), H.from_device(shard.buf.lse), O_ref, L_ref)
