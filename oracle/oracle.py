"""Plain fp64 CPU oracle for dynamic tile-sparse global attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline / reference arm may import this module; the product
path (the C-ABI library and its Python binding) never does, and there is no
CPU fallback built on it.  It shares no code with the CUDA path: it reads the
same seeded inputs (bf16 bit patterns or float32), converts them exactly to
float64 and recomputes every step with numpy in the order the method states.

The method (what is computed, and where each step comes from):

* Global (cross-frame) attention in VGGT-style backbones: every query token of
  every one of S frames attends to all S*N tokens, at quadratic cost in the
  number of frames ("AVGGT: Rethinking Global Attention for Accelerating VGGT",
  technical summary, section 1 "O Problema"; "(Full) Attention is More Than
  You Need", the full-vs-sparse figure).
* Dynamic sparsity: keep only the most promising query-key interactions,
  chosen per input, per layer and per head ("SAF3R: Dynamic Sparse Attention
  for Feed-Forward 3D Reconstruction Transformers", abstract).  The generic
  mechanism used here is tile-sparse attention ("Zebra3D: Efficient Hybrid
  Foundation Models For Scalable 3D Reconstruction", abstract): tiles of
  queries and keys are summarised by their means, scored by a per-head dot
  product, and each query tile keeps its top-k key tiles.
* Kept always: the query's own frame (frame attention is the cheap local
  case, AVGGT section 2.B.1, and the diagonal/self term is preserved, AVGGT
  section 2.B.2 "Preservacao Diagonal") and the special camera/register
  tokens of every frame (AVGGT section 2.B.2: all queries and special tokens
  are kept).
* Landmarks: unselected key tiles are not dropped but summarised (Zebra3D
  abstract, "landmark summaries to preserve unselected context"; AVGGT
  section 2.B.2 approximates discarded columns by a mean key/value pair).
  Each unselected tile j contributes one token (mean K, mean V) whose logit
  carries +ln(c_j), c_j the number of key rows it stands for, so that it
  weighs as c_j copies of the mean key.

Readings taken where the pages are silent (all listed in the design notes):
tiles are frame aligned (the last tile of a frame is partial); k counts only
tiles outside the own frame; sink keys are excluded from tiles and attended
exactly once each; sink rows are ordinary queries; the score is the plain dot
product of fp64 tile means (no 1/sqrt(d), which does not change a ranking);
equal scores go to the lower key-tile index; the landmark bias is added after
the softmax scale.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


# ----------------------------------------------------------------------------- inputs

def to_f64(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) or float32 to float64."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if a.dtype in (np.float32, np.float64):
        return a.astype(np.float64)
    raise TypeError("unsupported input dtype %s" % a.dtype)


# ----------------------------------------------------------------------------- geometry

@dataclasses.dataclass(frozen=True)
class Geometry:
    """Frame-aligned tiling of S frames x N tokens (token t = s*N + n)."""
    frames: int
    tokens: int
    tile: int
    n_sink: int

    @property
    def L(self) -> int:
        return self.frames * self.tokens

    @property
    def tpf(self) -> int:
        return -(-self.tokens // self.tile)

    @property
    def nt(self) -> int:
        return self.frames * self.tpf

    def frame_of_tile(self, j: int) -> int:
        return j // self.tpf

    def tile_rows(self, j: int) -> np.ndarray:
        """All token indices of tile j (its query rows)."""
        f, slot = divmod(j, self.tpf)
        lo = slot * self.tile
        hi = min(self.tokens, lo + self.tile)
        return f * self.tokens + np.arange(lo, hi)

    def tile_key_rows(self, j: int) -> np.ndarray:
        """Token indices of tile j that enter tile visits and key pooling (non-sink)."""
        f, slot = divmod(j, self.tpf)
        lo = max(slot * self.tile, self.n_sink)
        hi = min(self.tokens, slot * self.tile + self.tile)
        if hi <= lo:
            return np.zeros((0,), np.int64)
        return f * self.tokens + np.arange(lo, hi)

    def sink_rows(self) -> np.ndarray:
        """Every frame's special tokens, frame-major (the sink segment order)."""
        return np.array([s * self.tokens + n for s in range(self.frames) for n in range(self.n_sink)],
                        dtype=np.int64)

    def key_count(self, j: int) -> int:
        """Number of non-sink rows of tile j (the landmark multiplicity c_j)."""
        return len(self.tile_key_rows(j))

    def own_frame_tiles(self, i: int) -> np.ndarray:
        f = self.frame_of_tile(i)
        return np.arange(f * self.tpf, (f + 1) * self.tpf)


# ----------------------------------------------------------------------------- step 1: pooling

def pool(g: Geometry, q: np.ndarray, k: np.ndarray, v: np.ndarray | None = None):
    """Tile means (Zebra3D abstract: tiles summarised by landmarks; AVGGT 2.B.2 mean K-V pair).

    q, k, v: [BH][L][d] float64.  Returns (q_bar, k_bar, v_bar, cnt, sink_k, sink_v):
      q_bar[h, j] = mean of q over all rows of tile j;
      k_bar[h, j] = mean of k over the non-sink rows of tile j (0 if there are none);
      v_bar likewise (None when v is None);
      cnt[j]      = number of non-sink rows of tile j;
      sink_k/v    = the sink rows of every frame, frame-major, [BH][S*n_sink][d].
    """
    bh, L, d = q.shape
    assert L == g.L
    nt = g.nt
    q_bar = np.zeros((bh, nt, d))
    k_bar = np.zeros((bh, nt, d))
    v_bar = None if v is None else np.zeros((bh, nt, v.shape[2]))
    cnt = np.zeros((nt,), np.int64)
    for j in range(nt):
        rq = g.tile_rows(j)
        rk = g.tile_key_rows(j)
        q_bar[:, j] = q[:, rq].mean(axis=1)
        cnt[j] = len(rk)
        if len(rk):
            k_bar[:, j] = k[:, rk].mean(axis=1)
            if v is not None:
                v_bar[:, j] = v[:, rk].mean(axis=1)
    sr = g.sink_rows()
    sink_k = k[:, sr]
    sink_v = None if v is None else v[:, sr]
    return q_bar, k_bar, v_bar, cnt, sink_k, sink_v


# ----------------------------------------------------------------------------- step 2: scores

def scores(q_bar: np.ndarray, k_bar: np.ndarray) -> np.ndarray:
    """Per-head tile scores s[h, i, j] = q_bar[h, i] . k_bar[h, j] (SAF3R abstract: rank the
    query-key interactions by promise; the dot product of tile means is the ranking signal)."""
    return np.einsum("hid,hjd->hij", q_bar, k_bar)


# ----------------------------------------------------------------------------- step 3: selection

def candidates(g: Geometry, i: int) -> np.ndarray:
    """Key tiles that query tile i may choose: outside its own frame, with a non-sink row.
    (Which rows of a tile are sinks depends only on the tile's slot within its frame.)"""
    slot_has_key = np.array([g.key_count(slot) > 0 for slot in range(g.tpf)], dtype=bool)
    j = np.arange(g.nt, dtype=np.int64)
    return j[(j // g.tpf != g.frame_of_tile(i)) & slot_has_key[j % g.tpf]]


def select_row(g: Geometry, s_row: np.ndarray, i: int, k: int) -> np.ndarray:
    """Kept key tiles of query tile i, ascending.

    Forced: every tile of the query's own frame (AVGGT 2.B.1 frame attention and the preserved
    diagonal of 2.B.2).  Chosen: the k highest-scoring tiles among the candidates, ordered by
    (score descending, index ascending); all of them when k >= their number.
    """
    forced = g.own_frame_tiles(i)
    cand = candidates(g, i)
    kk = max(0, min(int(k), len(cand)))
    order = np.lexsort((cand, -s_row[cand]))  # primary: -score, secondary: index
    chosen = cand[order[:kk]]
    return np.sort(np.concatenate([forced, chosen]))


def select(g: Geometry, s: np.ndarray, k: int):
    """kept[h][i] for every head h and query tile i."""
    bh = s.shape[0]
    return [[select_row(g, s[h, i], i, k) for i in range(g.nt)] for h in range(bh)]


def select_per_head(g: Geometry, s: np.ndarray, k_per_head):
    """kept[h][i] when head h keeps its own budget k_per_head[h] of candidate tiles.

    Attention sparsity differs from head to head, and budgets are set per head from offline
    profiling and online adaptation ("SAF3R" abstract).  The selection rule of each head is
    the single-budget rule; a budget at or above the candidate count makes that head dense.
    """
    return [[select_row(g, s[h, i], i, int(k_per_head[h])) for i in range(g.nt)] for h in range(s.shape[0])]


# ----------------------------------------------------------------------------- per-head budgets

def candidate_entropy(g: Geometry, s_row: np.ndarray, i: int, scale: float) -> float:
    """Entropy (natural log) of the softmax of scale * s_row over the candidate tiles of query
    tile i: H = -sum_j p_j ln p_j with p_j = exp(x_j) / sum_c exp(x_c), x = scale * s.
    Written as ln Z - sum_j p_j (x_j - m) with m = max x and Z = sum_j exp(x_j - m), which is
    the same quantity without a logarithm of a vanishing p.  No candidate: 0."""
    cand = candidates(g, i)
    if len(cand) == 0:
        return 0.0
    x = scale * s_row[cand]
    m = x.max()
    w = np.exp(x - m)
    z = w.sum()
    return float(np.log(z) - (w / z * (x - m)).sum())


def head_budgets(g: Geometry, q_bar: np.ndarray, k_bar: np.ndarray, scale: float, beta: float,
                 k_lo: int, k_hi: int):
    """Per-head budgets from an online statistic of the head's own pooled scores.

    Heads differ in how concentrated their attention is, and the budget of each head is
    adapted online ("SAF3R" abstract: per-head sparsity from offline profiling and online
    adaptation).  The statistic of head h is the mean perplexity of its query tiles,
        P_h = (1/nt) sum_i exp(H_i),
    H_i the entropy of the softmax of scale * s_ij over the candidate tiles j of tile i (0 for
    a tile without candidates, so that it adds nothing): the effective number of candidates the
    tile-level attention spreads over.  The budget keeps that many tiles, scaled by beta:
        k_h = min(k_hi, max(k_lo, floor(beta * P_h + 1/2))).
    Uniform scores give P_h = the candidate count (every candidate kept when beta >= 1); one
    dominant candidate per row gives P_h -> 1.  Returns (P [bh], k [bh] int64)."""
    s = scores(q_bar, k_bar)
    bh = s.shape[0]
    perp = np.zeros((bh,))
    for h in range(bh):
        tot = 0.0
        for i in range(g.nt):
            tot += np.exp(candidate_entropy(g, s[h, i], i, scale)) if len(candidates(g, i)) else 0.0
        perp[h] = tot / g.nt
    k = np.minimum(k_hi, np.maximum(k_lo, np.floor(beta * perp + 0.5))).astype(np.int64)
    return perp, k


def budget_matches(perp_ref: float, beta: float, k_lo: int, k_hi: int, got: int, rel: float = 1e-4) -> bool:
    """A GPU budget computed in f32 is accepted iff it equals the fp64 rule's, or beta * P lies
    within rel (relative) of a rounding boundary n + 1/2 and the GPU took the other side."""
    want = int(min(k_hi, max(k_lo, np.floor(beta * perp_ref + 0.5))))
    if got == want:
        return True
    x = beta * perp_ref
    frac_dist = abs((x - 0.5) - np.round(x - 0.5))
    return abs(got - want) == 1 and frac_dist <= rel * max(1.0, abs(x))


def max_kept(g: Geometry, k: int) -> int:
    """Length of every kept list: own-frame tiles plus min(k, candidates)."""
    n_cand = (g.frames - 1) * sum(1 for slot in range(g.tpf) if g.key_count(slot) > 0)
    return g.tpf + max(0, min(int(k), n_cand))


# ----------------------------------------------------------------------------- step 4: attention

def _softmax_rows(logits: np.ndarray, values: np.ndarray):
    """Two-pass softmax of each row of `logits` applied to `values`; returns (O, LSE)."""
    m = logits.max(axis=1, keepdims=True)
    w = np.exp(logits - m)
    z = w.sum(axis=1, keepdims=True)
    o = (w @ values) / z
    lse = (m + np.log(z))[:, 0]
    return o, lse


def attend_tile(g: Geometry, q: np.ndarray, k: np.ndarray, v: np.ndarray, h: int, i: int,
                kept: np.ndarray, scale: float, landmark: bool = False,
                k_bar: np.ndarray | None = None, v_bar: np.ndarray | None = None,
                cnt: np.ndarray | None = None):
    """Outputs of the query rows of tile i of head h on a given kept list.

    Attended set of every row (Zebra3D abstract; AVGGT 2.B.2):
      (i)   the non-sink rows of every listed tile,
      (ii)  every frame's sink rows, once each,
      (iii) in landmark mode, one token (k_bar_j, v_bar_j) with logit bias ln(cnt_j)
            for every unlisted tile j with cnt_j > 0.
    Logits are scale * q.k (+ bias); softmax is taken over the whole attended set.
    """
    rows = g.tile_rows(i)
    key_rows = [g.tile_key_rows(int(j)) for j in kept]
    key_rows.append(g.sink_rows())
    kr = np.concatenate(key_rows) if key_rows else np.zeros((0,), np.int64)
    qh = q[h, rows]
    logits = scale * (qh @ k[h, kr].T)
    values = v[h, kr]
    if landmark:
        listed = np.zeros((g.nt,), bool)
        listed[np.asarray(kept, np.int64)] = True
        lm = np.nonzero((~listed) & (cnt > 0))[0]
        if len(lm):
            lm_logits = scale * (qh @ k_bar[h, lm].T) + np.log(cnt[lm].astype(np.float64))[None, :]
            logits = np.concatenate([logits, lm_logits], axis=1)
            values = np.concatenate([values, v_bar[h, lm]], axis=0)
    return rows, _softmax_rows(logits, values)


def attend(g: Geometry, q: np.ndarray, k: np.ndarray, v: np.ndarray, kept, scale: float,
           landmark: bool = False, k_bar=None, v_bar=None, cnt=None, items=None):
    """Full output O [BH][L][d] and LSE [BH][L] (NaN where a row was not computed).

    `kept[h][i]` is the list for query tile i of head h; `items`, if given, restricts the
    work to those (h, i) pairs.
    """
    bh, L, _ = q.shape
    O = np.full((bh, L, v.shape[2]), np.nan)
    LSE = np.full((bh, L), np.nan)
    todo = items if items is not None else [(h, i) for h in range(bh) for i in range(g.nt)]
    for h, i in todo:
        rows, (o, lse) = attend_tile(g, q, k, v, h, i, kept[h][i], scale, landmark, k_bar, v_bar, cnt)
        O[h, rows] = o
        LSE[h, rows] = lse
    return O, LSE


def attend_bruteforce(g: Geometry, q, k, v, kept, scale: float, landmark: bool = False,
                      k_bar=None, v_bar=None, cnt=None):
    """Same outputs as `attend`, built as one explicit [L x (L + nt)] bias matrix per head
    (0 where a pair is attended, -inf where it is not, ln cnt_j on landmark columns) followed
    by a full-row softmax.  For tiny shapes only; it shares no bookkeeping with `attend`
    beyond the tile geometry."""
    bh, L, _ = q.shape
    nt = g.nt
    O = np.zeros((bh, L, v.shape[2]))
    LSE = np.zeros((bh, L))
    for h in range(bh):
        bias = np.full((L, L + nt), -np.inf)
        for t in range(L):
            s_t, n_t = divmod(t, g.tokens)
            i = s_t * g.tpf + n_t // g.tile  # query tile of row t
            listed = set(int(x) for x in kept[h][i])
            for u in range(L):
                s_u, n_u = divmod(u, g.tokens)
                if n_u < g.n_sink:
                    bias[t, u] = 0.0  # special tokens: attended once by everyone
                    continue
                j = s_u * g.tpf + n_u // g.tile
                if j in listed:
                    bias[t, u] = 0.0
            if landmark:
                for j in range(nt):
                    if j not in listed and cnt[j] > 0:
                        bias[t, L + j] = math.log(cnt[j])
        keys = k[h] if not landmark else np.concatenate([k[h], k_bar[h]], axis=0)
        vals = v[h] if not landmark else np.concatenate([v[h], v_bar[h]], axis=0)
        if not landmark:
            bias = bias[:, :L]
        logits = scale * (q[h] @ keys.T) + bias
        O[h], LSE[h] = _softmax_rows(logits, vals)
    return O, LSE


# ----------------------------------------------------------------------------- backward of step 4

def attend_backward(g: Geometry, q: np.ndarray, k: np.ndarray, v: np.ndarray, kept, do: np.ndarray,
                    scale: float, landmark: bool = False, cnt: np.ndarray | None = None, items=None):
    """Gradients (dq, dk, dv) of sum(do * O) for O = attend(g, q, k, v, kept, scale, landmark).

    The kept lists are constants of the layer call: selection is piecewise constant in its
    inputs, so no gradient flows through pooling and scoring into it.  The landmark tokens
    are differentiable functions of K and V (the tile means), so their gradients flow back
    to the tile's non-sink rows, each receiving 1/c_j of it ("Zebra3D", abstract: landmark
    summaries of unselected tiles, used for post-conversion training).
    Per query tile, with the attended keys and values stacked in the forward's order:
      P  = softmax(logits)                 (the forward's probabilities)
      dV_att += P^T dO,   dP = dO V_att^T, Dr = rowsum(dO * O)
      dS = P * (dP - Dr),  dQ = scale dS K_att,  dK_att += scale dS^T Q.
    `items` restricts the query tiles taken as in `attend` (the gradients then cover only
    their contributions).
    """
    bh, L, d = q.shape
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    if landmark:
        _, k_bar, v_bar, cnt_p, _, _ = pool(g, q, k, v)
        cnt = cnt_p if cnt is None else cnt
        dk_bar = np.zeros((bh, g.nt, d))
        dv_bar = np.zeros((bh, g.nt, v.shape[2]))
    todo = items if items is not None else [(h, i) for h in range(bh) for i in range(g.nt)]
    for h, i in todo:
        rows = g.tile_rows(i)
        kr = np.concatenate([g.tile_key_rows(int(j)) for j in kept[h][i]] + [g.sink_rows()])
        qh, doh = q[h, rows], do[h, rows]
        keys, vals = k[h, kr], v[h, kr]
        logits = scale * (qh @ keys.T)
        lm = np.zeros((0,), np.int64)
        if landmark:
            listed = np.zeros((g.nt,), bool)
            listed[np.asarray(kept[h][i], np.int64)] = True
            lm = np.nonzero((~listed) & (cnt > 0))[0]
            logits = np.concatenate([logits, scale * (qh @ k_bar[h, lm].T) + np.log(cnt[lm].astype(np.float64))],
                                    axis=1)
            keys = np.concatenate([keys, k_bar[h, lm]], axis=0)
            vals = np.concatenate([vals, v_bar[h, lm]], axis=0)
        m = logits.max(axis=1, keepdims=True)
        w = np.exp(logits - m)
        p = w / w.sum(axis=1, keepdims=True)
        o = p @ vals
        d_v = p.T @ doh
        dp = doh @ vals.T
        dr = (doh * o).sum(axis=1, keepdims=True)
        ds = p * (dp - dr)
        dq[h, rows] += scale * (ds @ keys)
        d_k = scale * (ds.T @ qh)
        n_rows = len(kr)
        np.add.at(dk[h], kr, d_k[:n_rows])
        np.add.at(dv[h], kr, d_v[:n_rows])
        if len(lm):
            dk_bar[h, lm] += d_k[n_rows:]
            dv_bar[h, lm] += d_v[n_rows:]
    if landmark:  # k_bar_j is the mean of the c_j non-sink rows of tile j
        for j in range(g.nt):
            rk = g.tile_key_rows(j)
            if len(rk):
                dk[:, rk] += dk_bar[:, j][:, None, :] / len(rk)
                dv[:, rk] += dv_bar[:, j][:, None, :] / len(rk)
    return dq, dk, dv


def dense_backward(q, k, v, do, scale: float):
    """Gradients of sum(do * O) for textbook dense attention (the sparsity-0 control)."""
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for h in range(q.shape[0]):
        lg = scale * (q[h] @ k[h].T)
        w = np.exp(lg - lg.max(axis=1, keepdims=True))
        p = w / w.sum(axis=1, keepdims=True)
        o = p @ v[h]
        dv[h] = p.T @ do[h]
        ds = p * (do[h] @ v[h].T - (do[h] * o).sum(axis=1, keepdims=True))
        dq[h] = scale * (ds @ k[h])
        dk[h] = scale * (ds.T @ q[h])
    return dq, dk, dv


# ----------------------------------------------------------------------------- subsampled global attention

def sga_kept(frames: int, tokens: int, n_special: int, grid_h: int, grid_w: int, s_h: int, s_w: int):
    """Boolean [S*N]: the key/value tokens a subsampled global attention layer keeps.

    Every frame is n_special special tokens followed by a grid_h x grid_w patch grid in
    row-major order.  Kept: all special tokens, and the patch at (r, c) when r is a multiple of
    s_h and c a multiple of s_w - one token per s_h x s_w window of the 2-D grid ("AVGGT",
    technical summary 2.B.2, "Estrategia de Grade": keys and values subsampled uniformly on a
    2-D grid; special tokens preserved).
    """
    if n_special + grid_h * grid_w != tokens:
        raise ValueError("tokens must be n_special + grid_h * grid_w")
    per = np.zeros((tokens,), bool)
    per[:n_special] = True
    r = np.arange(grid_h)[:, None]
    c = np.arange(grid_w)[None, :]
    per[n_special:] = ((r % s_h == 0) & (c % s_w == 0)).reshape(-1)
    return np.tile(per, frames)


def sga(q, k, v, frames: int, tokens: int, n_special: int, grid_h: int, grid_w: int, s_h: int, s_w: int,
        scale: float, rows=None):
    """Subsampled global attention ("AVGGT", technical summary 2.B.2, SGA).

    Every query attends to the kept tokens (sga_kept), to its own key (the diagonal is
    preserved explicitly), and to one extra key/value pair standing for the discarded columns:
    the mean key and mean value of the discarded tokens of all frames - for a query whose own
    token is discarded, all of them except itself, since its column is kept as the diagonal -
    with a logit bias of ln(count), so that the pair weighs as the columns it replaces (the
    aggregated response of the discarded columns is kept).  Returns (O [bh][L][d], LSE [bh][L]);
    with `rows` (token indices) only those query rows are computed (the others stay zero).
    """
    bh, L, _ = q.shape
    kept = sga_kept(frames, tokens, n_special, grid_h, grid_w, s_h, s_w)
    disc = np.nonzero(~kept)[0]
    kidx = np.nonzero(kept)[0]
    n_d = len(disc)
    O = np.zeros((bh, L, v.shape[2]))
    LSE = np.zeros((bh, L))
    for h in range(bh):
        k_sum = k[h, disc].sum(axis=0)
        v_sum = v[h, disc].sum(axis=0)
        for t in (range(L) if rows is None else rows):
            own_disc = not kept[t]
            keys = [k[h, kidx]]
            vals = [v[h, kidx]]
            logits = [scale * (k[h, kidx] @ q[h, t])]
            if own_disc:  # the diagonal
                keys.append(k[h, t][None])
                vals.append(v[h, t][None])
                logits.append(np.array([scale * (k[h, t] @ q[h, t])]))
            c = n_d - (1 if own_disc else 0)
            if c > 0:  # the mean pair of the other discarded columns
                kb = (k_sum - (k[h, t] if own_disc else 0.0)) / c
                vb = (v_sum - (v[h, t] if own_disc else 0.0)) / c
                vals.append(vb[None])
                logits.append(np.array([scale * (kb @ q[h, t]) + math.log(c)]))
            lg = np.concatenate(logits)[None, :]
            o, lse = _softmax_rows(lg, np.concatenate(vals, axis=0))
            O[h, t], LSE[h, t] = o[0], lse[0]
    return O, LSE


def dense(q, k, v, scale: float):
    """Textbook dense softmax attention over all L keys (the sparsity-0 control)."""
    bh, L, _ = q.shape
    O = np.zeros((bh, L, v.shape[2]))
    LSE = np.zeros((bh, L))
    for h in range(bh):
        O[h], LSE[h] = _softmax_rows(scale * (q[h] @ k[h].T), v[h])
    return O, LSE


# ----------------------------------------------------------------------------- selection parity rule

def selection_matches(g: Geometry, s_row: np.ndarray, i: int, k: int, got: np.ndarray,
                      rel: float = 1e-4, floor: float = 1e-7):
    """Check a selected list against the oracle's for query tile i (s_row in fp64).

    Accepted iff it is ascending without repeats, has the oracle's size, contains every
    own-frame tile, and every swap against the oracle's choice is between near-equal scores:
    for a in got\\ref and b in ref\\got, s_b - s_a <= rel*max(|s_a|,|s_b|) + floor*max|s_row|.
    Returns (ok, message).
    """
    ref = select_row(g, s_row, i, k)
    got = np.asarray(got, np.int64)
    if len(got) != len(ref):
        return False, "size %d != %d" % (len(got), len(ref))
    if len(got) > 1 and not np.all(np.diff(got) > 0):
        return False, "not strictly ascending"
    if not np.all(np.isin(g.own_frame_tiles(i), got)):
        return False, "own-frame tile missing"
    if got.min(initial=0) < 0 or got.max(initial=0) >= g.nt:
        return False, "index out of range"
    extra = np.setdiff1d(got, ref)
    missing = np.setdiff1d(ref, got)
    if len(extra) == 0:
        return True, "exact"
    smax = float(np.abs(s_row).max())
    for a in extra:
        for b in missing:
            sa, sb = float(s_row[a]), float(s_row[b])
            if sb - sa > rel * max(abs(sa), abs(sb)) + floor * smax:
                return False, "swap %d<->%d beyond tolerance (%.9g vs %.9g)" % (a, b, sa, sb)
    return True, "%d near-tie swaps" % len(extra)
