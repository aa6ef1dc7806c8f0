"""The seeded input generator: determinism and the recipe's structure."""
import numpy as np

import synth
from synth.workloads import ALL, TINY, VGGT_S16, Workload


def f32(a):
    return (a.astype(np.uint32) << 16).view(np.float32) if a.dtype == np.uint16 else a


def test_workload_budgets():
    got = {w.name: (w.tpf, w.nt, w.k, w.max_kept) for w in ALL}
    assert got["tiny_s4_n256"] == (4, 16, 4, 8)
    assert got["vggt_s16_n1374"] == (11, 176, 35, 46)
    assert got["vggt_s128_n1374"] == (11, 1408, 130, 141)
    assert got["vggt_s512_n1374_landmark"] == (11, 5632, 327, 338)
    assert got["vggt_s1024_n1374_streamed"] == (11, 11264, 327, 338)


def test_deterministic_and_seeded():
    a = synth.generate(TINY, threads=3)
    b = synth.generate(TINY, threads=1)
    for key in ("q", "k", "v", "point"):
        assert np.array_equal(a[key], b[key])
    c = synth.generate(TINY, seed=1)
    assert not np.array_equal(a["q"], c["q"])
    # heads are independent draws: fewer heads give a prefix of the same values
    d = synth.generate(TINY, heads=1)
    assert np.array_equal(d["v"][0], a["v"][0])


def test_tiny_recipe_statistics():
    d = synth.generate(TINY)
    q, k, v = d["q"], d["k"], d["v"]
    assert q.dtype == np.float32 and q.shape == (2, 1024, 64)
    assert (d["point"] >= 0).all() and d["point"].max() < 128     # every token tied, P = 128
    for a in (q, k, v):
        assert abs(a.mean()) < 0.02 and abs(a.std() - 1.0) < 0.02
    # tokens tied to the same point share 0.8 z: E[q.k] = 0.64 d for the same point, 0 otherwise
    p = d["point"]
    same = np.nonzero(p[:, None] == p[None, :])
    dots = np.einsum("td,td->t", q[0][same[0][:2000]], k[0][same[1][:2000]])
    assert abs(dots.mean() / 64 - 0.64) < 0.05


def test_vggt_recipe_structure():
    w = VGGT_S16.scaled(frames=4)
    d = synth.generate(w, heads=2)
    q, k = f32(d["q"]), f32(d["k"])
    n = np.arange(w.L) % w.tokens
    sink = n < w.n_sink
    assert (d["point"][sink] == -1).all()
    assert abs((d["point"][~sink] >= 0).mean() - 0.7) < 0.02
    assert abs(k[:, sink].std() - 4.0) < 0.15 and abs(k[:, ~sink].std() - 1.0) < 0.02
    assert abs(q[:, sink].std() - 1.0) < 0.1
    # bf16 output is round-to-nearest-even of the float value: low 16 bits of the float are gone
    assert d["q"].dtype == np.uint16


def test_visibility_window():
    w = Workload("win", 12, 40, 1, 8, 8, 0, "bf16", 1, False, False, 64, 3, 1.0)
    d = synth.generate(w)
    p = d["point"]
    frames_of = {}
    for t, pt in enumerate(p):
        if pt >= 0:
            frames_of.setdefault(int(pt), set()).add(t // w.tokens)
    assert frames_of
    assert max(max(f) - min(f) for f in frames_of.values()) <= w.window - 1


def test_head_shard_is_a_slice_of_the_full_draw():
    import numpy as np
    import synth
    from synth.workloads import TINY, VGGT_S16
    for w in (TINY, VGGT_S16.scaled(frames=2)):
        full = synth.generate(w, heads=4)
        part = synth.generate(w, heads=2, head0=1)
        for x in ("q", "k", "v"):
            assert np.array_equal(part[x], full[x][1:3])
        assert np.array_equal(part["point"], full["point"])
