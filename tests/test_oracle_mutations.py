"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins catch each one.

Every mutant below is a one-line slip of the kind that would silently corrupt
parity: a dropped term, a wrong sign, a swapped index, a transposed operand.
The pins in test_oracle_pins.py must fail for every one of them.
"""
import math

import numpy as np
import pytest

import tests.test_oracle_pins as pins
from oracle import oracle as orc

PIN_TESTS = [
    lambda: pins.test_pool_against_explicit_loops(),
    lambda: pins.test_pool_ignores_sink_keys(),
    lambda: pins.test_scores_closed_form(),
    lambda: pins.test_scores_not_transposed(),
    *[lambda s=s: pins.test_select_bruteforce_subsets(s) for s in range(3)],
    lambda: pins.test_select_per_head_bruteforce(),
    lambda: pins.test_select_edges(),
    lambda: pins.test_select_skips_keyless_tiles(),
    lambda: pins.test_attention_two_key_closed_form(),
    lambda: pins.test_attention_landmark_closed_form_weight(),
    *[lambda l=l, n=n, k=k: pins.test_list_mode_equals_explicit_mask(l, n, k)
      for l in (False, True) for n in (0, 1) for k in (1, 99)],
    lambda: pins.test_all_tiles_equals_textbook_dense(2),
    lambda: pins.test_weights_sum_to_one(True),
    lambda: pins.test_frame_permutation_equivariance(True),
    lambda: pins.test_landmarks_exact_when_tile_keys_are_identical(),
    lambda: pins.test_k0_is_frame_attention_plus_sinks(),
    lambda: pins.test_sga_kept_positions(),
    *[lambda a=a, b=b: pins.test_sga_exact_when_discarded_tokens_are_identical(a, b) for a, b in ((2, 2), (3, 2))],
    lambda: pins.test_backward_all_tiles_is_dense(2),
    lambda: pins.test_backward_landmarks_exact_when_tile_rows_are_identical(),
    lambda: pins.test_backward_matches_finite_differences(True, 1, 1),
    lambda: pins.test_candidate_entropy_two_candidates_closed_form(),
    lambda: pins.test_candidate_entropy_bruteforce_excludes_own_frame_and_keyless_tiles(),
    lambda: pins.test_head_budgets_uniform_scores_give_the_candidate_count(),
    lambda: pins.test_head_budgets_mean_of_perplexities_bruteforce(),
]


def _some_pin_fails():
    for t in PIN_TESTS:
        try:
            t()
        except (AssertionError, ValueError, IndexError):
            return True
    return False


# ---- mutants -----------------------------------------------------------------------------

_pool = orc.pool
_attend_tile = orc.attend_tile
_select_row = orc.select_row
_softmax_rows = orc._softmax_rows
_tile_key_rows = orc.Geometry.tile_key_rows


def pool_with_sinks(g, q, k, v=None):
    qb, kb, vb, cnt, sk, sv = _pool(g, q, k, v)
    for j in range(g.nt):  # slip: key means over all rows, sinks included
        kb[:, j] = k[:, g.tile_rows(j)].mean(axis=1)
    return qb, kb, vb, cnt, sk, sv


def scores_transposed(q_bar, k_bar):
    return np.einsum("hjd,hid->hij", q_bar, k_bar)


def select_ties_high(g, s_row, i, k):
    forced = g.own_frame_tiles(i)
    cand = orc.candidates(g, i)
    kk = max(0, min(int(k), len(cand)))
    order = np.lexsort((-cand, -s_row[cand]))  # slip: higher index wins ties
    return np.sort(np.concatenate([forced, cand[order[:kk]]]))


def select_counts_own_frame(g, s_row, i, k):
    forced = g.own_frame_tiles(i)
    return _select_row(g, s_row, i, max(0, k - len(forced)))  # slip: k includes own frame


def select_no_force(g, s_row, i, k):
    cand = np.arange(g.nt)  # slip: own frame competes instead of being forced
    order = np.lexsort((cand, -s_row[cand]))
    return np.sort(cand[order[:orc.max_kept(g, k)]])


_select_per_head = orc.select_per_head


def per_head_first_budget(g, s, k_per_head):
    return _select_per_head(g, s, [k_per_head[0]] * s.shape[0])  # slip: one budget for every head


def per_head_budgets_shifted(g, s, k_per_head):
    ks = list(k_per_head)
    return _select_per_head(g, s, ks[1:] + ks[:1])  # slip: budget of the next head


_sga_kept = orc.sga_kept


def sga_kept_offset(frames, tokens, n_special, grid_h, grid_w, s_h, s_w):
    kept = _sga_kept(frames, tokens, n_special, grid_h, grid_w, s_h, s_w)
    per = kept[:tokens].copy()
    patches = per[n_special:].reshape(grid_h, grid_w)
    per[n_special:] = np.roll(patches, (s_h - 1, s_w - 1), axis=(0, 1)).reshape(-1)  # slip: last of each window
    return np.tile(per, frames)


def sga_kept_no_specials(frames, tokens, n_special, grid_h, grid_w, s_h, s_w):
    kept = _sga_kept(frames, tokens, n_special, grid_h, grid_w, s_h, s_w).reshape(frames, tokens)
    kept[:, :n_special] = False  # slip: special tokens subsampled away
    return kept.reshape(-1)


def _sga_variant(count_mode="exclude", keep_diagonal=True, bias=True):
    def sga(q, k, v, frames, tokens, n_special, grid_h, grid_w, s_h, s_w, scale):
        bh, L, _ = q.shape
        kept = orc.sga_kept(frames, tokens, n_special, grid_h, grid_w, s_h, s_w)
        disc = np.nonzero(~kept)[0]
        kidx = np.nonzero(kept)[0]
        O = np.zeros((bh, L, v.shape[2]))
        LSE = np.zeros((bh, L))
        for h in range(bh):
            for t in range(L):
                own = not kept[t]
                keys, vals = [k[h, kidx]], [v[h, kidx]]
                if own and keep_diagonal:
                    keys.append(k[h, t][None]); vals.append(v[h, t][None])
                others = disc[disc != t] if count_mode == "exclude" else disc
                lg = [scale * (np.concatenate(keys) @ q[h, t])]
                if len(others):
                    kb, vb = k[h, others].mean(axis=0), v[h, others].mean(axis=0)
                    lg.append(np.array([scale * (kb @ q[h, t]) + (math.log(len(others)) if bias else 0.0)]))
                    vals.append(vb[None])
                o, lse = orc._softmax_rows(np.concatenate(lg)[None], np.concatenate(vals))
                O[h, t], LSE[h, t] = o[0], lse[0]
        return O, LSE
    return sga


def _attend_variant(bias_sign=1.0, drop_scale=False, drop_sinks=False, bias_inside_scale=False):
    def attend_tile(g, q, k, v, h, i, kept, scale, landmark=False, k_bar=None, v_bar=None, cnt=None):
        rows = g.tile_rows(i)
        kr = [g.tile_key_rows(int(j)) for j in kept]
        if not drop_sinks:
            kr.append(g.sink_rows())
        kr = np.concatenate(kr)
        sc = 1.0 if drop_scale else scale
        logits = sc * (q[h, rows] @ k[h, kr].T)
        values = v[h, kr]
        if landmark:
            listed = np.zeros((g.nt,), bool)
            listed[np.asarray(kept, np.int64)] = True
            lm = np.nonzero((~listed) & (cnt > 0))[0]
            if len(lm):
                b = bias_sign * np.log(cnt[lm].astype(float))[None, :]
                if bias_inside_scale:
                    lml = sc * (q[h, rows] @ k_bar[h, lm].T + b)
                else:
                    lml = sc * (q[h, rows] @ k_bar[h, lm].T) + b
                logits = np.concatenate([logits, lml], axis=1)
                values = np.concatenate([values, v_bar[h, lm]], axis=0)
        return rows, orc._softmax_rows(logits, values)
    return attend_tile


def softmax_lse_without_max(logits, values):
    o, lse = _softmax_rows(logits, values)
    m = logits.max(axis=1)
    return o, lse - m  # slip: forgot to add the running max back


def softmax_no_normalise(logits, values):
    m = logits.max(axis=1, keepdims=True)
    w = np.exp(logits - m)
    return w @ values, (m + np.log(w.sum(axis=1, keepdims=True)))[:, 0]


def key_rows_keep_sinks(self, j):
    f, slot = divmod(j, self.tpf)
    lo = slot * self.tile  # slip: sink rows stay inside tile 0 of each frame
    hi = min(self.tokens, lo + self.tile)
    return f * self.tokens + np.arange(lo, hi)


def _backward_variant(drop_rowsum=False, share_whole=False, dk_unscaled=False, dq_from_values=False,
                      drop_lm_bias=False):
    def attend_backward(g, q, k, v, kept, do, scale, landmark=False, cnt=None, items=None):
        bh, L, d = q.shape
        dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
        if landmark:
            _, k_bar, v_bar, cnt, _, _ = orc.pool(g, q, k, v)
            dk_bar, dv_bar = np.zeros((bh, g.nt, d)), np.zeros((bh, g.nt, d))
        for h in range(bh):
            for i in range(g.nt):
                rows = g.tile_rows(i)
                kr = np.concatenate([g.tile_key_rows(int(j)) for j in kept[h][i]] + [g.sink_rows()])
                keys, vals = k[h, kr], v[h, kr]
                logits = scale * (q[h, rows] @ keys.T)
                lm = np.zeros((0,), np.int64)
                if landmark:
                    listed = np.zeros((g.nt,), bool)
                    listed[np.asarray(kept[h][i], np.int64)] = True
                    lm = np.nonzero((~listed) & (cnt > 0))[0]
                    b = 0.0 if drop_lm_bias else np.log(cnt[lm].astype(float))
                    logits = np.concatenate([logits, scale * (q[h, rows] @ k_bar[h, lm].T) + b], axis=1)
                    keys = np.concatenate([keys, k_bar[h, lm]])
                    vals = np.concatenate([vals, v_bar[h, lm]])
                w = np.exp(logits - logits.max(axis=1, keepdims=True))
                p = w / w.sum(axis=1, keepdims=True)
                dr = 0.0 if drop_rowsum else (do[h, rows] * (p @ vals)).sum(axis=1, keepdims=True)
                ds = p * (do[h, rows] @ vals.T - dr)
                dq[h, rows] += scale * (ds @ (vals if dq_from_values else keys))
                d_k = (1.0 if dk_unscaled else scale) * (ds.T @ q[h, rows])
                d_v = p.T @ do[h, rows]
                np.add.at(dk[h], kr, d_k[:len(kr)])
                np.add.at(dv[h], kr, d_v[:len(kr)])
                if len(lm):
                    dk_bar[h, lm] += d_k[len(kr):]
                    dv_bar[h, lm] += d_v[len(kr):]
        if landmark:
            for j in range(g.nt):
                rk = g.tile_key_rows(j)
                if len(rk):
                    c = 1 if share_whole else len(rk)
                    dk[:, rk] += dk_bar[:, j][:, None, :] / c
                    dv[:, rk] += dv_bar[:, j][:, None, :] / c
        return dq, dk, dv
    return attend_backward


_candidate_entropy = orc.candidate_entropy


def entropy_over_every_tile(g, s_row, i, scale):
    x = scale * s_row  # slip: own frame and keyless tiles enter the softmax
    m = x.max()
    w = np.exp(x - m)
    z = w.sum()
    return float(np.log(z) - (w / z * (x - m)).sum())


def entropy_unscaled(g, s_row, i, scale):
    return _candidate_entropy(g, s_row, i, 1.0)  # slip: temperature dropped


def entropy_base2(g, s_row, i, scale):
    return _candidate_entropy(g, s_row, i, scale) / math.log(2.0)  # slip: bits instead of nats


def head_budgets_exp_of_mean_entropy(g, q_bar, k_bar, scale, beta, k_lo, k_hi):
    s = orc.scores(q_bar, k_bar)
    perp = np.array([math.exp(np.mean([orc.candidate_entropy(g, s[h, i], i, scale) for i in range(g.nt)]))
                     for h in range(s.shape[0])])  # slip: exp of the mean entropy
    k = np.minimum(k_hi, np.maximum(k_lo, np.floor(beta * perp + 0.5))).astype(np.int64)
    return perp, k


MUTANTS = {
    "entropy_over_every_tile": ("candidate_entropy", entropy_over_every_tile),
    "entropy_unscaled": ("candidate_entropy", entropy_unscaled),
    "entropy_base2": ("candidate_entropy", entropy_base2),
    "budget_exp_of_mean_entropy": ("head_budgets", head_budgets_exp_of_mean_entropy),
    "bwd_rowsum_term_dropped": ("attend_backward", _backward_variant(drop_rowsum=True)),
    "bwd_landmark_gradient_not_shared": ("attend_backward", _backward_variant(share_whole=True)),
    "bwd_dk_unscaled": ("attend_backward", _backward_variant(dk_unscaled=True)),
    "bwd_dq_from_values": ("attend_backward", _backward_variant(dq_from_values=True)),
    "bwd_landmark_bias_dropped": ("attend_backward", _backward_variant(drop_lm_bias=True)),
    "pool_includes_sinks": ("pool", pool_with_sinks),
    "scores_transposed": ("scores", scores_transposed),
    "ties_to_higher_index": ("select_row", select_ties_high),
    "k_counts_own_frame": ("select_row", select_counts_own_frame),
    "own_frame_not_forced": ("select_row", select_no_force),
    "per_head_one_budget": ("select_per_head", per_head_first_budget),
    "per_head_budgets_shifted": ("select_per_head", per_head_budgets_shifted),
    "landmark_bias_negated": ("attend_tile", _attend_variant(bias_sign=-1.0)),
    "scale_dropped": ("attend_tile", _attend_variant(drop_scale=True)),
    "sinks_dropped": ("attend_tile", _attend_variant(drop_sinks=True)),
    "bias_inside_scale": ("attend_tile", _attend_variant(bias_inside_scale=True)),
    "lse_without_max": ("_softmax_rows", softmax_lse_without_max),
    "sga_grid_offset": ("sga_kept", sga_kept_offset),
    "sga_specials_dropped": ("sga_kept", sga_kept_no_specials),
    "sga_count_includes_own_column": ("sga", _sga_variant(count_mode="all")),
    "sga_diagonal_dropped": ("sga", _sga_variant(keep_diagonal=False)),
    "sga_no_count_bias": ("sga", _sga_variant(bias=False)),
    "softmax_not_normalised": ("_softmax_rows", softmax_no_normalise),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(orc, attr, fn)
    assert _some_pin_fails(), "mutant %s survived every pin" % name


def test_key_rows_mutant_is_caught(monkeypatch):
    monkeypatch.setattr(orc.Geometry, "tile_key_rows", key_rows_keep_sinks)
    assert _some_pin_fails()


def test_unmutated_oracle_passes_every_pin():
    assert not _some_pin_fails()
    assert math.isfinite(1.0)
