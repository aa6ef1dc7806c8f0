"""One sparse global-attention layer call: the four C-ABI steps on caller-visible buffers.

`SparseGlobalAttention` owns the intermediate device buffers (tile means,
scores or the streamed-selection block, kept lists, landmark workspace) as
torch tensors and runs

    sa_tile_pool -> sa_tile_scores (materialised mode only) -> sa_select_topk
                 -> sa_sparse_attn_fwd

on the current CUDA stream.  torch provides device memory and streams only;
every step runs in libsa's kernels.
"""
from __future__ import annotations

import dataclasses

from . import sa


@dataclasses.dataclass
class Buffers:
    q_pool: object
    k_pool: object
    v_pool: object
    k_cnt: object
    sink_k: object
    sink_v: object
    scores: object
    sel_ws: object
    kept_idx: object
    kept_cnt: object
    attn_ws: object
    o: object
    lse: object


class SparseGlobalAttention:
    """Dynamic tile-sparse global attention for bh heads of S frames x N tokens (d = 64).

    k          key tiles chosen per query tile beyond its own frame's tiles
    landmark   fold every unselected tile into one mean-K/mean-V token (+ln count bias)
    streamed   select without materialising the [bh][nt][nt] score matrix
    """

    def __init__(self, bh: int, frames: int, tokens: int, k: int, tile: int = 128, n_sink: int = 5,
                 dtype: str = "bf16", landmark: bool = False, streamed: bool = False, head_dim: int = 64,
                 device=None, with_lse: bool = True):
        import torch
        self.shape = sa.shape(bh, frames, tokens, head_dim, tile, n_sink, dtype)
        self.k = int(k)
        self.landmark = bool(landmark)
        self.streamed = bool(streamed)
        self.nt = sa.sa_num_tiles(self.shape)
        if self.nt < 0:
            raise ValueError("invalid shape")
        self.max_kept = sa.sa_max_kept(self.shape, self.k)
        self.bh, self.frames, self.tokens, self.d = bh, frames, tokens, head_dim
        self.L = frames * tokens
        dev = torch.device(device if device is not None else "cuda")
        self.device = dev
        tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
        self.dtype = tdt
        f32, i32 = torch.float32, torch.int32
        nt = self.nt
        sel_bytes = sa.sa_select_workspace_size(self.shape, self.streamed)
        attn_bytes = sa.sa_sparse_attn_workspace_size(self.shape, self.landmark)
        self.buf = Buffers(
            q_pool=torch.empty((bh, nt, head_dim), dtype=f32, device=dev),
            k_pool=torch.empty((bh, nt, head_dim), dtype=f32, device=dev),
            v_pool=torch.empty((bh, nt, head_dim), dtype=f32, device=dev) if self.landmark else None,
            k_cnt=torch.empty((nt,), dtype=i32, device=dev),
            sink_k=torch.empty((bh, max(1, frames * n_sink), head_dim), dtype=tdt, device=dev),
            sink_v=torch.empty((bh, max(1, frames * n_sink), head_dim), dtype=tdt, device=dev),
            scores=None if self.streamed else torch.empty((bh, nt, nt), dtype=f32, device=dev),
            sel_ws=torch.empty((max(1, sel_bytes),), dtype=torch.uint8, device=dev) if sel_bytes else None,
            kept_idx=torch.empty((bh, nt, self.max_kept), dtype=i32, device=dev),
            kept_cnt=torch.empty((bh, nt), dtype=i32, device=dev),
            attn_ws=torch.empty((attn_bytes,), dtype=torch.uint8, device=dev) if attn_bytes else None,
            o=torch.empty((bh, self.L, head_dim), dtype=tdt, device=dev),
            lse=torch.empty((bh, self.L), dtype=f32, device=dev) if with_lse else None,
        )

    # individual steps (each one C call) ---------------------------------------------------------
    def pool(self, q, k, v, stream=None):
        b = self.buf
        sa.sa_tile_pool(self.shape, q, k, v, b.q_pool, b.k_pool, b.v_pool, b.k_cnt, b.sink_k, b.sink_v, stream)

    def score(self, stream=None):
        if not self.streamed:
            sa.sa_tile_scores(self.shape, self.buf.q_pool, self.buf.k_pool, self.buf.scores, stream)

    def select(self, stream=None):
        b = self.buf
        sa.sa_select_topk(self.shape, b.scores, b.q_pool, b.k_pool, self.k, b.kept_idx, b.kept_cnt,
                          self.max_kept, b.sel_ws, stream)

    def attend(self, q, k, v, stream=None):
        b = self.buf
        sa.sa_sparse_attn_fwd(self.shape, q, k, v, b.kept_idx, b.kept_cnt, self.max_kept, b.sink_k, b.sink_v,
                              self.landmark, b.k_pool, b.v_pool, b.k_cnt, b.attn_ws, b.o, b.lse, stream)

    def forward(self, q, k, v, stream=None):
        """Run the whole layer call on device tensors [bh][S*N][d]; returns (O, LSE) buffers."""
        self.pool(q, k, v, stream)
        self.score(stream)
        self.select(stream)
        self.attend(q, k, v, stream)
        return self.buf.o, self.buf.lse

    __call__ = forward

    def launches_per_call(self) -> int:
        """Kernel launches libsa makes for one forward (for launch accounting)."""
        n = 1  # pooling
        if self.streamed:
            rows = sa.sa_select_workspace_size(self.shape, True) // (4 * self.nt)
            n += 2 * self.bh * (-(-self.nt // rows))  # score block + select block
        else:
            n += 2  # scores + select
        n += 1  # attention
        if sa.sa_sparse_attn_workspace_size(self.shape, self.landmark) > 0:
            n += 1  # transposed V tiles
            if self.frames * self.shape.n_sink > 0:
                n += 1  # transposed sink V tiles
            if self.landmark:
                n += 1  # landmark tables
        return n


def dense_attention(q, k, v, frames: int, tokens: int, dtype: str = "bf16", with_lse: bool = True, stream=None):
    """Dense control on device tensors [bh][S*N][64]; returns (O, LSE)."""
    import torch
    bh = q.shape[0]
    shp = sa.shape(bh, frames, tokens, q.shape[2], 128, 0, dtype)
    o = torch.empty_like(q)
    lse = torch.empty((bh, frames * tokens), dtype=torch.float32, device=q.device) if with_lse else None
    nbytes = sa.sa_dense_attn_workspace_size(shp)
    ws = torch.empty((nbytes,), dtype=torch.uint8, device=q.device) if nbytes else None
    sa.sa_dense_attn_fwd(shp, q, k, v, ws, o, lse, stream)
    return o, lse


class DenseAttention:
    """Dense control with its workspace allocated once (for repeated calls at one shape)."""

    def __init__(self, bh: int, frames: int, tokens: int, dtype: str = "bf16", head_dim: int = 64, device=None):
        import torch
        self.shape = sa.shape(bh, frames, tokens, head_dim, 128, 0, dtype)
        dev = torch.device(device if device is not None else "cuda")
        nbytes = sa.sa_dense_attn_workspace_size(self.shape)
        self.ws = torch.empty((nbytes,), dtype=torch.uint8, device=dev) if nbytes else None
        tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
        self.o = torch.empty((bh, frames * tokens, head_dim), dtype=tdt, device=dev)
        self.lse = torch.empty((bh, frames * tokens), dtype=torch.float32, device=dev)

    def __call__(self, q, k, v, stream=None):
        sa.sa_dense_attn_fwd(self.shape, q, k, v, self.ws, self.o, self.lse, stream)
        return self.o, self.lse
