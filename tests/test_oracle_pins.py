"""Pins for the fp64 oracle against facts that do not come from the oracle itself.

Each check fixes the oracle to something independent: exact bit patterns,
hand-derived closed forms, brute-force enumeration on tiny inputs, textbook
identities (softmax weights sum to one, dense attention as the all-tiles
case, frame attention as the k = 0 case) and symmetry (frame permutation).
"""
import itertools
import math

import numpy as np
import pytest

from oracle import oracle as orc


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


# ----------------------------------------------------------------------------- inputs, geometry

def test_bf16_widening_exact():
    bits = np.array([0x3F80, 0xC000, 0x3E80, 0x0000, 0x8000, 0x7F7F, 0x0001], np.uint16)
    got = orc.to_f64(bits)
    want = [1.0, -2.0, 0.25, 0.0, -0.0, 3.3895313892515355e38, 9.183549615799121e-41]
    assert got.tolist() == want


def test_geometry_vggt_tiles():
    g = orc.Geometry(frames=3, tokens=1374, tile=128, n_sink=5)
    assert g.tpf == 11 and g.nt == 33
    assert len(g.tile_rows(10)) == 94                # partial last tile of a frame
    assert g.key_count(0) == 123 and g.key_count(1) == 128 and g.key_count(10) == 94
    # query rows partition the tokens; key rows plus sinks partition them too
    q_rows = np.concatenate([g.tile_rows(j) for j in range(g.nt)])
    assert np.array_equal(np.sort(q_rows), np.arange(g.L))
    k_rows = np.concatenate([g.tile_key_rows(j) for j in range(g.nt)] + [g.sink_rows()])
    assert np.array_equal(np.sort(k_rows), np.arange(g.L))
    assert g.tile_rows(11)[0] == 1374                # tiles restart at every frame


# ----------------------------------------------------------------------------- pooling

def test_pool_against_explicit_loops():
    g = orc.Geometry(frames=2, tokens=7, tile=3, n_sink=2)
    q, k, v = rnd((2, g.L, 4), 1), rnd((2, g.L, 4), 2), rnd((2, g.L, 4), 3)
    qb, kb, vb, cnt, sk, sv = orc.pool(g, q, k, v)
    for h in range(2):
        for j in range(g.nt):
            f, slot = divmod(j, g.tpf)
            sq = [0.0] * 4
            sk_ = [0.0] * 4
            sv_ = [0.0] * 4
            nq = nk = 0
            for n in range(slot * 3, min(7, slot * 3 + 3)):
                t = f * 7 + n
                nq += 1
                for e in range(4):
                    sq[e] += q[h, t, e]
                if n >= 2:
                    nk += 1
                    for e in range(4):
                        sk_[e] += k[h, t, e]
                        sv_[e] += v[h, t, e]
            assert cnt[j] == nk
            np.testing.assert_allclose(qb[h, j], [x / nq for x in sq], rtol=1e-14, atol=1e-15)
            if nk:
                np.testing.assert_allclose(kb[h, j], [x / nk for x in sk_], rtol=1e-14, atol=1e-15)
                np.testing.assert_allclose(vb[h, j], [x / nk for x in sv_], rtol=1e-14, atol=1e-15)
    # the sink segment is frame-major: frame 0's tokens 0,1 then frame 1's tokens 0,1
    np.testing.assert_array_equal(sk[:, 2], k[:, 7])
    np.testing.assert_array_equal(sv[:, 3], v[:, 8])


def test_pool_ignores_sink_keys():
    g = orc.Geometry(frames=1, tokens=8, tile=4, n_sink=1)
    k = np.ones((1, 8, 2))
    k[0, 0] = 1e6  # a sink key must not leak into its tile's mean
    _, kb, _, cnt, _, _ = orc.pool(g, np.zeros_like(k), k)
    assert cnt.tolist() == [3, 4]
    assert np.array_equal(kb[0], np.ones((2, 2)))


# ----------------------------------------------------------------------------- scores

def test_scores_closed_form():
    # tile means along coordinate axes: s_ij = alpha_i * beta_j if axes match else 0
    g = orc.Geometry(frames=2, tokens=4, tile=2, n_sink=0)
    d = 4
    q = np.zeros((1, g.L, d))
    k = np.zeros((1, g.L, d))
    alpha = [0.5, -2.0, 3.0, 1.5]
    beta = [4.0, 0.25, -1.0, 2.0]
    axes_q = [0, 1, 2, 1]
    axes_k = [1, 1, 0, 3]
    for j in range(g.nt):
        for t in g.tile_rows(j):
            q[0, t, axes_q[j]] = alpha[j]
            k[0, t, axes_k[j]] = beta[j]
    qb, kb, _, _, _, _ = orc.pool(g, q, k)
    s = orc.scores(qb, kb)
    for i in range(4):
        for j in range(4):
            want = alpha[i] * beta[j] if axes_q[i] == axes_k[j] else 0.0
            assert s[0, i, j] == want


def test_scores_not_transposed():
    qb = np.array([[[1.0, 0.0], [0.0, 1.0]]])
    kb = np.array([[[0.0, 3.0], [5.0, 0.0]]])
    s = orc.scores(qb, kb)
    assert s[0].tolist() == [[0.0, 5.0], [3.0, 0.0]]


# ----------------------------------------------------------------------------- selection

def _is_topk(s, cand, subset):
    # subset is the top-k iff every member beats every non-member by (score desc, index asc)
    inside = set(subset)
    for a in inside:
        for b in cand:
            if b in inside:
                continue
            if not (s[a] > s[b] or (s[a] == s[b] and a < b)):
                return False
    return True


@pytest.mark.parametrize("seed", range(6))
def test_select_bruteforce_subsets(seed):
    g = orc.Geometry(frames=3, tokens=6, tile=2, n_sink=0)  # tpf 3, nt 9
    rng = np.random.default_rng(seed)
    s = rng.integers(-3, 4, size=g.nt).astype(float)  # many exact ties on purpose
    for i in range(g.nt):
        cand = [j for j in range(g.nt) if j // 3 != i // 3]
        for k in range(0, len(cand) + 2):
            kk = min(k, len(cand))
            winners = [c for c in itertools.combinations(cand, kk) if _is_topk(s, cand, c)]
            assert len(winners) == 1
            want = sorted(list(winners[0]) + [j for j in range(g.nt) if j // 3 == i // 3])
            assert orc.select_row(g, s, i, k).tolist() == want


def test_select_per_head_bruteforce():
    """Per-head budgets: each head's lists are the brute-force top-k of that head's row."""
    g = orc.Geometry(frames=3, tokens=6, tile=2, n_sink=0)  # tpf 3, nt 9, 6 candidates
    rng = np.random.default_rng(11)
    budgets = [0, 2, 5, 99]
    s = rng.integers(-2, 3, size=(len(budgets), g.nt, g.nt)).astype(float)
    kept = orc.select_per_head(g, s, budgets)
    for h, k in enumerate(budgets):
        for i in range(g.nt):
            cand = [j for j in range(g.nt) if j // 3 != i // 3]
            kk = min(k, len(cand))
            winners = [c for c in itertools.combinations(cand, kk) if _is_topk(s[h, i], cand, c)]
            own = [j for j in range(g.nt) if j // 3 == i // 3]
            assert kept[h][i].tolist() == sorted(list(winners[0]) + own)


def test_selection_is_nested_in_the_budget():
    """With the (score desc, index asc) order, a larger budget only adds tiles."""
    g = orc.Geometry(frames=4, tokens=10, tile=4, n_sink=1)  # tpf 3, nt 12
    rng = np.random.default_rng(5)
    s = rng.integers(-3, 4, size=(g.nt, g.nt)).astype(float)
    for i in range(g.nt):
        prev = set(orc.select_row(g, s[i], i, 0).tolist())
        for k in range(1, g.nt + 2):
            cur = set(orc.select_row(g, s[i], i, k).tolist())
            assert prev <= cur and len(cur) - len(prev) <= 1
            prev = cur


def test_select_edges():
    g = orc.Geometry(frames=4, tokens=4, tile=2, n_sink=0)  # tpf 2, nt 8
    s = np.zeros(g.nt)
    assert orc.select_row(g, s, 5, 0).tolist() == [4, 5]                 # k = 0: own frame only
    assert orc.select_row(g, s, 5, 100).tolist() == list(range(8))      # k >= candidates: all
    assert orc.select_row(g, s, 5, 3).tolist() == [0, 1, 2, 4, 5]       # all equal: lowest index
    s = np.array([9.0, 1, 2, 3, 4, 5, 6, -1])
    assert orc.select_row(g, s, 0, 2).tolist() == [0, 1, 5, 6]          # own frame forced even if low
    assert orc.max_kept(g, 3) == 5 and orc.max_kept(g, 99) == 8


def test_select_skips_keyless_tiles():
    g = orc.Geometry(frames=2, tokens=4, tile=2, n_sink=2)  # slot 0 of each frame is all sinks
    s = np.array([100.0, 1.0, 50.0, 2.0])
    assert orc.select_row(g, s, 0, 1).tolist() == [0, 1, 3]
    assert orc.max_kept(g, 5) == 3


def test_selection_rule_accepts_near_ties_only():
    g = orc.Geometry(frames=2, tokens=8, tile=2, n_sink=0)  # tpf 4, nt 8
    s = np.array([0, 0, 0, 0, 1.0, 0.5, 0.5 * (1 - 5e-5), 0.1])
    ok, _ = orc.selection_matches(g, s, 0, 2, np.array([0, 1, 2, 3, 4, 5]))
    assert ok
    ok, msg = orc.selection_matches(g, s, 0, 2, np.array([0, 1, 2, 3, 4, 6]))
    assert ok and "swap" in msg
    ok, _ = orc.selection_matches(g, s, 0, 2, np.array([0, 1, 2, 3, 4, 7]))
    assert not ok
    ok, _ = orc.selection_matches(g, s, 0, 2, np.array([0, 1, 2, 4, 5, 6]))
    assert not ok  # own-frame tile 3 missing


# ----------------------------------------------------------------------------- attention

def test_attention_two_key_closed_form():
    # logits 0 and ln 3 give weights 1/4 and 3/4; LSE = ln 4
    g = orc.Geometry(frames=1, tokens=2, tile=2, n_sink=0)
    d = 4
    scale = 0.5
    q = np.zeros((1, 2, d))
    q[0, :, 0] = 1.0
    k = np.zeros((1, 2, d))
    k[0, 1, 0] = math.log(3.0) / scale
    v = np.array([[[1.0, 0, 0, 0], [0, 1.0, 0, 8.0]]])
    O, LSE = orc.attend(g, q, k, v, [[np.array([0])]], scale)
    np.testing.assert_allclose(O[0, 0], [0.25, 0.75, 0, 6.0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(LSE[0], [math.log(4.0)] * 2, rtol=0, atol=1e-15)


def test_attention_landmark_closed_form_weight():
    # one unlisted tile of c identical key rows acts as c copies: weight c*e^x / (c*e^x + e^y)
    g = orc.Geometry(frames=2, tokens=3, tile=3, n_sink=0)  # tpf 1: tile 0 = frame 0, tile 1 = frame 1
    d = 2
    scale = 1.0
    q = np.zeros((1, 6, d))
    q[0, :, 0] = 1.0
    k = np.zeros((1, 6, d))
    k[0, 0:3, 0] = [0.0, 0.3, -0.2]   # own frame (listed)
    k[0, 3:6, 0] = 0.7                # frame 1, unlisted, identical rows
    v = rnd((1, 6, d), 5)
    qb, kb, vb, cnt, _, _ = orc.pool(g, q, k, v)
    O, _ = orc.attend(g, q, k, v, [[np.array([0]), np.array([1])]], scale, landmark=True,
                      k_bar=kb, v_bar=vb, cnt=cnt)
    w_own = np.exp([0.0, 0.3, -0.2])
    w_lm = 3 * math.exp(0.7)
    want = (w_own @ v[0, 0:3] + w_lm * v[0, 3:6].mean(axis=0)) / (w_own.sum() + w_lm)
    np.testing.assert_allclose(O[0, 0], want, rtol=1e-14)


def _tiny_case(seed, frames=3, tokens=5, tile=2, n_sink=1, bh=2, d=4):
    g = orc.Geometry(frames, tokens, tile, n_sink)
    q, k, v = rnd((bh, g.L, d), seed), rnd((bh, g.L, d), seed + 1), rnd((bh, g.L, d), seed + 2)
    return g, q, k, v


@pytest.mark.parametrize("landmark", [False, True])
@pytest.mark.parametrize("n_sink", [0, 1, 2])
@pytest.mark.parametrize("kk", [0, 1, 3, 99])
def test_list_mode_equals_explicit_mask(landmark, n_sink, kk):
    g, q, k, v = _tiny_case(10 + n_sink, n_sink=n_sink)
    scale = 0.37
    qb, kb, vb, cnt, _, _ = orc.pool(g, q, k, v)
    kept = orc.select(g, orc.scores(qb, kb), kk)
    O1, L1 = orc.attend(g, q, k, v, kept, scale, landmark, kb, vb, cnt)
    O2, L2 = orc.attend_bruteforce(g, q, k, v, kept, scale, landmark, kb, vb, cnt)
    np.testing.assert_allclose(O1, O2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(L1, L2, rtol=0, atol=1e-12)


def _textbook_row(qr, K, V, scale):
    # one row, pure-Python loops with math.exp
    logits = [scale * sum(a * b for a, b in zip(qr, kr)) for kr in K]
    m = max(logits)
    w = [math.exp(x - m) for x in logits]
    z = sum(w)
    return [sum(wi * V[t][e] for t, wi in enumerate(w)) / z for e in range(len(V[0]))], m + math.log(z)


@pytest.mark.parametrize("n_sink", [0, 2])
def test_all_tiles_equals_textbook_dense(n_sink):
    g, q, k, v = _tiny_case(20, n_sink=n_sink)
    scale = 0.5
    qb, kb, vb, cnt, _, _ = orc.pool(g, q, k, v)
    kept = orc.select(g, orc.scores(qb, kb), 10 ** 6)
    for landmark in (False, True):  # no tile is unlisted, so landmark mode changes nothing
        O, LSE = orc.attend(g, q, k, v, kept, scale, landmark, kb, vb, cnt)
        for h in range(q.shape[0]):
            for t in range(g.L):
                o, lse = _textbook_row(q[h, t], k[h].tolist(), v[h].tolist(), scale)
                np.testing.assert_allclose(O[h, t], o, rtol=0, atol=1e-12)
                assert abs(LSE[h, t] - lse) < 1e-12
    Od, Ld = orc.dense(q, k, v, scale)
    np.testing.assert_allclose(O, Od, rtol=0, atol=1e-12)


@pytest.mark.parametrize("landmark", [False, True])
def test_weights_sum_to_one(landmark):
    g, q, k, _ = _tiny_case(30, frames=4, tokens=6, tile=2, n_sink=1)
    ones = np.ones((q.shape[0], g.L, 3))
    qb, kb, vb, cnt, _, _ = orc.pool(g, q, k, ones)
    kept = orc.select(g, orc.scores(qb, kb), 2)
    O, _ = orc.attend(g, q, k, ones, kept, 0.7, landmark, kb, vb, cnt)
    np.testing.assert_allclose(O, 1.0, rtol=0, atol=1e-12)
    # with one-hot values the outputs are the weights themselves: non-negative, summing to 1
    L = g.L
    onehot = np.broadcast_to(np.eye(L)[None], (q.shape[0], L, L)).copy()
    qb, kb, vb, cnt, _, _ = orc.pool(g, q, k, onehot)
    O, _ = orc.attend(g, q, k, onehot, kept, 0.7, landmark, kb, vb, cnt)
    assert O.min() >= 0.0
    np.testing.assert_allclose(O.sum(axis=2), 1.0, rtol=0, atol=1e-12)


@pytest.mark.parametrize("landmark", [False, True])
def test_frame_permutation_equivariance(landmark):
    g, q, k, v = _tiny_case(40, frames=5, tokens=5, tile=2, n_sink=1, bh=2, d=4)
    perm = np.array([3, 0, 4, 1, 2])  # new frame f holds old frame perm[f]
    tok = np.concatenate([np.arange(p * g.tokens, (p + 1) * g.tokens) for p in perm])

    def run(q, k, v):
        qb, kb, vb, cnt, _, _ = orc.pool(g, q, k, v)
        s = orc.scores(qb, kb)
        kept = orc.select(g, s, 2)
        return kept, orc.attend(g, q, k, v, kept, 0.4, landmark, kb, vb, cnt)

    kept_a, (Oa, La) = run(q, k, v)
    kept_b, (Ob, Lb) = run(q[:, tok], k[:, tok], v[:, tok])
    np.testing.assert_allclose(Ob, Oa[:, tok], rtol=0, atol=1e-12)
    np.testing.assert_allclose(Lb, La[:, tok], rtol=0, atol=1e-12)
    # kept sets map through the permutation: tile (f, slot) -> (perm^-1[f], slot)
    inv = np.argsort(perm)
    for h in range(2):
        for i in range(g.nt):
            f, slot = divmod(i, g.tpf)
            ia = perm[f] * g.tpf + slot
            mapped = sorted(int(inv[j // g.tpf] * g.tpf + j % g.tpf) for j in kept_a[h][ia])
            assert kept_b[h][i].tolist() == mapped


def test_landmarks_exact_when_tile_keys_are_identical():
    # every tile's non-sink keys equal one vector -> c_j copies are summarised exactly,
    # so landmark mode reproduces dense attention for any selection (partial tiles included)
    g = orc.Geometry(frames=4, tokens=7, tile=3, n_sink=1)  # counts 2,3,1 per frame
    d = 3
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, g.L, d))
    v = rng.standard_normal((1, g.L, d))
    k = np.zeros((1, g.L, d))
    for j in range(g.nt):
        k[0, g.tile_key_rows(j)] = rng.standard_normal(d)
    k[0, g.sink_rows()] = rng.standard_normal((len(g.sink_rows()), d))
    qb, kb, vb, cnt, _, _ = orc.pool(g, q, k, v)
    assert sorted(set(cnt.tolist())) == [1, 2, 3]
    kept = orc.select(g, orc.scores(qb, kb), 1)
    O, LSE = orc.attend(g, q, k, v, kept, 0.6, True, kb, vb, cnt)
    Od, Ld = orc.dense(q, k, v, 0.6)
    np.testing.assert_allclose(O, Od, rtol=0, atol=1e-12)
    np.testing.assert_allclose(LSE, Ld, rtol=0, atol=1e-12)


def test_k0_is_frame_attention_plus_sinks():
    g, q, k, v = _tiny_case(50, frames=3, tokens=6, tile=4, n_sink=2, bh=1)
    qb, kb, vb, cnt, _, _ = orc.pool(g, q, k, v)
    kept = orc.select(g, orc.scores(qb, kb), 0)
    O, _ = orc.attend(g, q, k, v, kept, 0.3)
    sinks = [s * 6 + n for s in range(3) for n in range(2)]
    for t in range(g.L):
        f = t // 6
        keys = [f * 6 + n for n in range(2, 6)] + sinks
        o, _ = _textbook_row(q[0, t], k[0, keys].tolist(), v[0, keys].tolist(), 0.3)
        np.testing.assert_allclose(O[0, t], o, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- subsampled global attention

def test_sga_kept_positions():
    # one frame: 2 special tokens, then a 3 x 5 grid; stride (2, 2) keeps rows 0, 2 and columns 0, 2, 4
    kept = orc.sga_kept(frames=2, tokens=2 + 15, n_special=2, grid_h=3, grid_w=5, s_h=2, s_w=2)
    per = [0, 1] + [2 + r * 5 + c for r in (0, 2) for c in (0, 2, 4)]
    assert np.nonzero(kept)[0].tolist() == per + [17 + j for j in per]


@pytest.mark.parametrize("n_special,gh,gw", [(0, 3, 4), (2, 4, 5)])
def test_sga_stride_one_is_dense(n_special, gh, gw):
    rng = np.random.default_rng(3)
    S, N = 2, n_special + gh * gw
    q, k, v = (rng.standard_normal((2, S * N, 8)) for _ in range(3))
    O, LSE = orc.sga(q, k, v, S, N, n_special, gh, gw, 1, 1, 0.3)
    Od, Ld = orc.dense(q, k, v, 0.3)
    assert np.abs(O - Od).max() < 1e-12 and np.abs(LSE - Ld).max() < 1e-12


@pytest.mark.parametrize("s_h,s_w", [(2, 2), (3, 2), (4, 5)])
def test_sga_exact_when_discarded_tokens_are_identical(s_h, s_w):
    """The mean pair stands for the discarded columns exactly when they are all equal: then the
    layer equals dense attention (this pins the ln(count) bias, the diagonal, and the count
    excluding the query's own discarded column)."""
    rng = np.random.default_rng(4)
    S, ns, gh, gw = 3, 2, 5, 7
    N = ns + gh * gw
    q, k, v = (rng.standard_normal((2, S * N, 8)) for _ in range(3))
    kept = orc.sga_kept(S, N, ns, gh, gw, s_h, s_w)
    for h in range(2):
        k[h, ~kept] = rng.standard_normal(8)
        v[h, ~kept] = rng.standard_normal(8)
    O, LSE = orc.sga(q, k, v, S, N, ns, gh, gw, s_h, s_w, 0.25)
    Od, Ld = orc.dense(q, k, v, 0.25)
    assert np.abs(O - Od).max() < 1e-12 and np.abs(LSE - Ld).max() < 1e-12


def test_sga_row_subset_matches_full():
    """Computing only some query rows changes nothing for those rows and leaves the rest zero."""
    rng = np.random.default_rng(5)
    S, ns, gh, gw = 2, 3, 4, 6
    N = ns + gh * gw
    q, k, v = (rng.standard_normal((2, S * N, 8)) for _ in range(3))
    O, LSE = orc.sga(q, k, v, S, N, ns, gh, gw, 2, 3, 0.25)
    rows = [0, 4, 17, N + 5, 2 * N - 1]
    Os, Ls = orc.sga(q, k, v, S, N, ns, gh, gw, 2, 3, 0.25, rows=rows)
    assert np.array_equal(Os[:, rows], O[:, rows]) and np.array_equal(Ls[:, rows], LSE[:, rows])
    rest = np.setdiff1d(np.arange(S * N), rows)
    assert not Os[:, rest].any() and not Ls[:, rest].any()


# ----------------------------------------------------------------------------- backward of the attention

def _loss(g, q, k, v, kept, do, scale, landmark):
    """sum(do * O) of the forward, with the landmark means recomputed from the given k, v."""
    qb, kb, vb, cnt, _, _ = orc.pool(g, q, k, v)
    O, _ = orc.attend(g, q, k, v, kept, scale, landmark, kb, vb, cnt)
    return float((do * O).sum())


@pytest.mark.parametrize("landmark", [False, True])
@pytest.mark.parametrize("n_sink,kk", [(0, 1), (1, 1), (2, 0)])
def test_backward_matches_finite_differences(landmark, n_sink, kk):
    """Central differences of the forward (which the pins above fix) over every input
    coordinate; the kept lists are held fixed, as the backward treats them."""
    g, q, k, v = _tiny_case(60 + n_sink, frames=3, tokens=5, tile=2, n_sink=n_sink, bh=1, d=3)
    scale = 0.45
    qb, kb, _, _, _, _ = orc.pool(g, q, k, v)
    kept = orc.select(g, orc.scores(qb, kb), kk)
    do = rnd(q.shape, 77)
    dq, dk, dv = orc.attend_backward(g, q, k, v, kept, do, scale, landmark)
    eps = 1e-5
    for x, grad in ((q, dq), (k, dk), (v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            keep = x[idx]
            x[idx] = keep + eps
            lp = _loss(g, q, k, v, kept, do, scale, landmark)
            x[idx] = keep - eps
            lm = _loss(g, q, k, v, kept, do, scale, landmark)
            x[idx] = keep
            fd[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(grad, fd, rtol=0, atol=1e-8)


def test_dense_backward_matches_autograd():
    import torch
    rng = np.random.default_rng(8)
    q, k, v, do = (rng.standard_normal((2, 11, 5)) for _ in range(4))
    dq, dk, dv = orc.dense_backward(q, k, v, do, 0.3)
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    o = torch.softmax(0.3 * tq @ tk.transpose(1, 2), dim=-1) @ tv
    (o * torch.tensor(do)).sum().backward()
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("n_sink", [0, 2])
def test_backward_all_tiles_is_dense(n_sink):
    g, q, k, v = _tiny_case(70, frames=3, tokens=6, tile=4, n_sink=n_sink, bh=2, d=4)
    kept = [[np.arange(g.nt) for _ in range(g.nt)] for _ in range(2)]
    do = rnd(q.shape, 71)
    got = orc.attend_backward(g, q, k, v, kept, do, 0.4)
    want = orc.dense_backward(q, k, v, do, 0.4)
    for a, b in zip(got, want):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_backward_landmarks_exact_when_tile_rows_are_identical():
    """Every tile's non-sink K rows equal one vector and its V rows another: the landmark of
    an unselected tile then stands exactly for its rows in the forward and in every gradient
    (the ln(c_j) bias and the 1/c_j share of the mean's gradient), so the gradients are the
    dense ones for any selection.  With only the K rows identical, dq and dv stay dense and
    dk keeps the dense sum over each tile's rows (a landmark spreads its share evenly)."""
    g = orc.Geometry(frames=4, tokens=7, tile=3, n_sink=1)  # counts 2, 3, 1 per frame
    d = 3
    rng = np.random.default_rng(9)
    q = rng.standard_normal((1, g.L, d))
    do = rng.standard_normal((1, g.L, d))
    k = rng.standard_normal((1, g.L, d))
    v = rng.standard_normal((1, g.L, d))
    for j in range(g.nt):
        k[0, g.tile_key_rows(j)] = rng.standard_normal(d)
    qb, kb, _, _, _, _ = orc.pool(g, q, k, v)
    kept = orc.select(g, orc.scores(qb, kb), 1)
    dq, dk, dv = orc.attend_backward(g, q, k, v, kept, do, 0.6, landmark=True)
    dq_d, dk_d, dv_d = orc.dense_backward(q, k, v, do, 0.6)
    np.testing.assert_allclose(dq, dq_d, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, dv_d, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk[0, g.sink_rows()], dk_d[0, g.sink_rows()], rtol=0, atol=1e-12)
    for j in range(g.nt):
        rk = g.tile_key_rows(j)
        np.testing.assert_allclose(dk[0, rk].sum(axis=0), dk_d[0, rk].sum(axis=0), rtol=0, atol=1e-12)
    for j in range(g.nt):
        v[0, g.tile_key_rows(j)] = rng.standard_normal(d)
    _, dk, _ = orc.attend_backward(g, q, k, v, kept, do, 0.6, landmark=True)
    _, dk_d, _ = orc.dense_backward(q, k, v, do, 0.6)
    np.testing.assert_allclose(dk, dk_d, rtol=0, atol=1e-12)


def test_backward_restricted_items_complete_what_they_cover():
    """Running only some query tiles gives the full backward's dq on those tiles, and the full
    dk, dv on a key tile's non-sink rows when every query tile that lists it is included (the
    sampled comparisons at large sizes rely on both)."""
    g, q, k, v = _tiny_case(80, frames=4, tokens=9, tile=4, n_sink=1, bh=1, d=3)
    qb, kb, _, _, _, _ = orc.pool(g, q, k, v)
    kept = orc.select(g, orc.scores(qb, kb), 2)
    do = rnd(q.shape, 81)
    dq, dk, dv = orc.attend_backward(g, q, k, v, kept, do, 0.5)
    tiles = [0, 5, g.nt - 1]
    dq_s, _, _ = orc.attend_backward(g, q, k, v, kept, do, 0.5, items=[(0, i) for i in tiles])
    rows = np.concatenate([g.tile_rows(i) for i in tiles])
    np.testing.assert_allclose(dq_s[0, rows], dq[0, rows], rtol=0, atol=1e-14)
    for j in (1, 6):
        users = [i for i in range(g.nt) if j in set(kept[0][i].tolist())]
        assert 0 < len(users) < g.nt
        _, dk_s, dv_s = orc.attend_backward(g, q, k, v, kept, do, 0.5, items=[(0, i) for i in users])
        kr = g.tile_key_rows(j)
        np.testing.assert_allclose(dk_s[0, kr], dk[0, kr], rtol=0, atol=1e-14)
        np.testing.assert_allclose(dv_s[0, kr], dv[0, kr], rtol=0, atol=1e-14)


# ----------------------------------------------------------------------------- per-head budgets

def _entropy_by_hand(probs):
    return -sum(p * math.log(p) for p in probs if p > 0.0)


def test_candidate_entropy_two_candidates_closed_form():
    """Three frames of one tile each: every query tile has exactly two candidates, whose softmax
    entropy is written out with math.exp / math.log."""
    g = orc.Geometry(frames=3, tokens=4, tile=4, n_sink=0)  # tpf 1, nt 3
    s = np.array([0.3, -1.2, 2.5])
    for i, tau in ((0, 0.7), (1, 2.0), (2, 0.1)):
        x = [tau * s[j] for j in range(3) if j != i]
        z = math.exp(x[0]) + math.exp(x[1])
        want = _entropy_by_hand([math.exp(x[0]) / z, math.exp(x[1]) / z])
        assert abs(orc.candidate_entropy(g, s, i, tau) - want) < 1e-12


def test_candidate_entropy_bruteforce_excludes_own_frame_and_keyless_tiles():
    g = orc.Geometry(frames=4, tokens=7, tile=3, n_sink=3)  # slot 0 of every frame is all sinks
    rng = np.random.default_rng(21)
    for i in range(g.nt):
        s = rng.standard_normal(g.nt) * 3
        cand = [j for j in range(g.nt) if j // g.tpf != i // g.tpf and (j % g.tpf) != 0]
        z = sum(math.exp(0.5 * s[j]) for j in cand)
        want = _entropy_by_hand([math.exp(0.5 * s[j]) / z for j in cand])
        assert abs(orc.candidate_entropy(g, s, i, 0.5) - want) < 1e-12


def test_head_budgets_uniform_scores_give_the_candidate_count():
    """Identical key means make every score of a row equal: the softmax is uniform, its
    perplexity is the number of candidates, and beta = 1 keeps all of them (the dense budget)."""
    g = orc.Geometry(frames=5, tokens=300, tile=128, n_sink=5)  # 3 slots, all holding keys
    rng = np.random.default_rng(3)
    qb = rng.standard_normal((2, g.nt, 8))
    kb = np.repeat(rng.standard_normal((2, 1, 8)), g.nt, axis=1)
    n_cand = (g.frames - 1) * g.tpf
    perp, k = orc.head_budgets(g, qb, kb, 0.9, 1.0, 0, 10_000)
    assert np.allclose(perp, n_cand, rtol=0, atol=1e-9)
    assert k.tolist() == [n_cand, n_cand]
    _, k = orc.head_budgets(g, qb, kb, 0.9, 0.5, 0, 10_000)
    assert k.tolist() == [n_cand // 2] * 2                 # floor(beta * P + 1/2), P = 12
    _, k = orc.head_budgets(g, qb, kb, 0.9, 1.0, 0, 7)
    assert k.tolist() == [7, 7]                            # clamped above
    _, k = orc.head_budgets(g, qb, kb, 0.9, 0.01, 5, 100)
    assert k.tolist() == [5, 5]                            # clamped below


def test_head_budgets_one_dominant_candidate():
    """One candidate far above the rest in every row: perplexity 1, whatever the head."""
    g = orc.Geometry(frames=3, tokens=8, tile=4, n_sink=0)  # tpf 2, nt 6, 4 candidates per row
    qb = np.zeros((1, g.nt, 2))
    qb[0, :, 0] = 1.0
    kb = np.zeros((1, g.nt, 2))
    kb[0, [0, 2, 4], 0] = [200.0, 150.0, 100.0]  # each row's best candidate beats the next by >= 50
    perp, k = orc.head_budgets(g, qb, kb, 1.0, 3.0, 0, 99)
    assert abs(perp[0] - 1.0) < 1e-12
    assert k[0] == 3


def test_head_budgets_mean_of_perplexities_bruteforce():
    g = orc.Geometry(frames=3, tokens=5, tile=2, n_sink=1)  # tpf 3, slot 0 holds 1 key row
    rng = np.random.default_rng(8)
    qb, kb = rng.standard_normal((3, g.nt, 4)), rng.standard_normal((3, g.nt, 4))
    perp, k = orc.head_budgets(g, qb, kb, 0.8, 0.7, 1, 6)
    for h in range(3):
        tot = 0.0
        for i in range(g.nt):
            cand = [j for j in range(g.nt) if j // 3 != i // 3]
            x = [0.8 * sum(qb[h, i, e] * kb[h, j, e] for e in range(4)) for j in cand]
            z = sum(math.exp(v) for v in x)
            tot += math.exp(_entropy_by_hand([math.exp(v) / z for v in x]))
        assert abs(perp[h] - tot / g.nt) < 1e-10
        assert k[h] == min(6, max(1, math.floor(0.7 * tot / g.nt + 0.5)))


def test_budget_rule_accepts_rounding_boundary_only():
    assert orc.budget_matches(10.2, 1.0, 0, 99, 10)
    assert not orc.budget_matches(10.2, 1.0, 0, 99, 11)
    assert orc.budget_matches(10.5 * (1 + 2e-5), 1.0, 0, 99, 10)   # f32 may round 10.50002 down
    assert orc.budget_matches(10.5 * (1 - 2e-5), 1.0, 0, 99, 11)
    assert not orc.budget_matches(10.5 * (1 + 2e-3), 1.0, 0, 99, 10)
