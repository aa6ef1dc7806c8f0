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


@dataclasses.dataclass
class GradBuffers:
    ws: object
    dq: object
    dk: object
    dv: object


class SparseGlobalAttention:
    """Dynamic tile-sparse global attention for bh heads of S frames x N tokens (d = 64).

    k          key tiles chosen per query tile beyond its own frame's tiles: one budget for every
               head, or a sequence of bh per-head budgets (a budget at or above the candidate
               count makes that head dense)
    adaptive   None, or a dict(temperature=, beta=, k_lo=) that sets every head's budget on the
               device from the spread of its own pooled scores (sa_head_budgets) before each
               selection; k is then the largest budget (k_hi); temperature defaults to tile/sqrt(d)
    landmark   fold every unselected tile into one mean-K/mean-V token (+ln count bias)
    streamed   select without materialising the [bh][nt][nt] score matrix
    """

    def __init__(self, bh: int, frames: int, tokens: int, k: int, tile: int = 128, n_sink: int = 5,
                 dtype: str = "bf16", landmark: bool = False, streamed: bool = False, head_dim: int = 64,
                 device=None, with_lse: bool = True, adaptive=None):
        import torch
        self.shape = sa.shape(bh, frames, tokens, head_dim, tile, n_sink, dtype)
        self.adaptive = None
        if adaptive is not None:
            if not (isinstance(k, int) or getattr(k, "ndim", None) == 0):
                raise ValueError("with adaptive budgets k is the single largest budget")
            ad = dict(adaptive)
            self.adaptive = (float(ad.get("temperature", tile / head_dim ** 0.5)), float(ad.get("beta", 1.0)),
                             int(ad.get("k_lo", 0)), int(k))
        if isinstance(k, (int,)) or getattr(k, "ndim", None) == 0:
            self.k, self.k_per_head = int(k), None
        else:
            ks = [int(x) for x in k]
            if len(ks) != bh or min(ks) < 0:
                raise ValueError("k needs one non-negative budget per head")
            self.k, self.k_per_head = max(ks), ks
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
        self.k_head = (torch.tensor(self.k_per_head, dtype=torch.int32, device=dev)
                       if self.k_per_head is not None else None)
        self.perplexity = None
        self.budget_ws = None
        if self.adaptive is not None:
            self.k_head = torch.zeros((bh,), dtype=torch.int32, device=dev)
            self.perplexity = torch.zeros((bh,), dtype=torch.float32, device=dev)
            self.budget_ws = torch.empty((sa.sa_head_budget_workspace_size(self.shape),), dtype=torch.uint8,
                                         device=dev)
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
        self.grad = None  # backward buffers, allocated by the first backward call

    # individual steps (each one C call) ---------------------------------------------------------
    def pool(self, q, k, v, stream=None):
        b = self.buf
        sa.sa_tile_pool(self.shape, q, k, v, b.q_pool, b.k_pool, b.v_pool, b.k_cnt, b.sink_k, b.sink_v, stream)

    def score(self, stream=None):
        if not self.streamed:
            sa.sa_tile_scores(self.shape, self.buf.q_pool, self.buf.k_pool, self.buf.scores, stream)

    def budgets(self, stream=None):
        """Adaptive mode: every head's budget from its own pooled scores (one C call)."""
        if self.adaptive is not None:
            tau, beta, k_lo, k_hi = self.adaptive
            sa.sa_head_budgets(self.shape, self.buf.q_pool, self.buf.k_pool, tau, beta, k_lo, k_hi, self.k_head,
                               self.perplexity, self.budget_ws, stream)

    def select(self, stream=None):
        b = self.buf
        self.budgets(stream)
        if self.k_head is None:
            sa.sa_select_topk(self.shape, b.scores, b.q_pool, b.k_pool, self.k, b.kept_idx, b.kept_cnt,
                              self.max_kept, b.sel_ws, stream)
        else:
            sa.sa_select_topk_per_head(self.shape, b.scores, b.q_pool, b.k_pool, self.k_head, self.k, b.kept_idx,
                                       b.kept_cnt, self.max_kept, b.sel_ws, stream)

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

    def capture(self, q, k, v):
        """Record one whole layer call on these input tensors as a CUDA graph and return it.

        `g.replay()` then re-runs every launch of the call (pooling, scoring, selection -- a few
        hundred launches in streamed mode -- and attention) from one host call, on the current
        stream; new inputs are written into q, k, v in place before a replay, and the results
        land in `self.buf.o` / `self.buf.lse` as with `forward`.  The library allocates nothing
        and every step is stream-ordered, so the call is captured as it runs.  One eager call
        comes first so that no kernel attribute is set inside the capture."""
        import torch
        self.forward(q, k, v)
        torch.cuda.current_stream(self.device).synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.forward(q, k, v)
        return g

    def backward(self, q, k, v, d_o, stream=None):
        """Gradients (dq, dk, dv) of sum(d_o * O) for the last forward on these q, k, v, with its
        kept lists held fixed; d_o is [bh][S*N][d] like O.  Needs the forward's LSE."""
        import torch
        b = self.buf
        if b.lse is None:
            raise ValueError("the backward needs the forward's LSE (with_lse=True)")
        if self.grad is None:
            nbytes = sa.sa_sparse_attn_bwd_workspace_size(self.shape, self.max_kept, self.landmark)
            if nbytes == 0:
                raise ValueError("no backward for this shape (bf16, tile 128, d 64 only)")
            dev = self.device
            self.grad = GradBuffers(
                ws=torch.empty((nbytes,), dtype=torch.uint8, device=dev),
                dq=torch.empty((self.bh, self.L, self.d), dtype=self.dtype, device=dev),
                dk=torch.empty((self.bh, self.L, self.d), dtype=self.dtype, device=dev),
                dv=torch.empty((self.bh, self.L, self.d), dtype=self.dtype, device=dev),
            )
        gr = self.grad
        sa.sa_sparse_attn_bwd(self.shape, q, k, v, b.o, b.lse, d_o, b.kept_idx, b.kept_cnt, self.max_kept,
                              b.sink_k, b.sink_v, self.landmark, b.k_pool, b.v_pool, b.k_cnt, gr.ws, gr.dq, gr.dk,
                              gr.dv, stream)
        return gr.dq, gr.dk, gr.dv

    def backward_launches(self) -> int:
        """Kernel launches libsa makes for one backward (memsets not counted)."""
        n = 1 + 3 + 3 + 3  # row terms; Q, dO, K transposes; list scan, plan, fill; dQ, dK/dV, finalize
        if self.frames * self.shape.n_sink > 0:
            n += 1  # transposed sink K tiles
        if self.landmark:
            n += 3  # landmark K and V tables, transposed landmark K chunks
        return n

    def launches_per_call(self) -> int:
        """Kernel launches libsa makes for one forward (for launch accounting)."""
        n = 1  # pooling
        if self.streamed:
            rows = sa.sa_select_workspace_size(self.shape, True) // (4 * self.nt)
            n += 2 * self.bh * (-(-self.nt // rows))  # score block + select block
        else:
            n += 2  # scores + select
        if self.adaptive is not None:
            n += 2  # per-head statistic + budgets
        n += 1  # attention
        if sa.sa_sparse_attn_workspace_size(self.shape, self.landmark) > 0:
            n += 1  # transposed V tiles
            if self.frames * self.shape.n_sink > 0:
                n += 1  # transposed sink V tiles
            if self.landmark:
                n += 1  # landmark tables
        return n


class HostPipeline:
    """Layer calls on host-resident (pinned) Q/K/V with the transfers overlapped.

    Two layer objects and two sets of device inputs alternate between calls; three streams
    carry the host-to-device copies, the four C-ABI steps and the device-to-host copy of O, so
    that the copy-in of call i+1 and the copy-out of call i-1 run while call i computes.
    `make_layer` builds one `SparseGlobalAttention`; inputs are [bh][L][d] host tensors.
    """

    def __init__(self, make_layer):
        import torch
        self.layers = [make_layer(), make_layer()]
        lay = self.layers[0]
        shape = (lay.bh, lay.L, lay.d)
        self.dev_in = [[torch.empty(shape, dtype=lay.dtype, device=lay.device) for _ in range(3)] for _ in range(2)]
        self.s_in = torch.cuda.Stream(lay.device)
        self.s_comp = torch.cuda.Stream(lay.device)
        self.s_out = torch.cuda.Stream(lay.device)
        self.ev_in = [torch.cuda.Event() for _ in range(2)]    # inputs of buffer set s are on the device
        self.ev_comp = [torch.cuda.Event() for _ in range(2)]  # the layer of set s has finished
        self.ev_out = [torch.cuda.Event() for _ in range(2)]   # O of set s has left the device
        self.calls = 0

    def submit(self, hq, hk, hv, ho):
        """Queue one call: hq, hk, hv pinned host inputs, ho the pinned host output."""
        import torch
        s = self.calls % 2
        self.calls += 1
        dq, dk, dv = self.dev_in[s]
        self.s_in.wait_event(self.ev_comp[s])  # the call two back has consumed these buffers
        with torch.cuda.stream(self.s_in):
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
        self.ev_in[s].record(self.s_in)
        self.s_comp.wait_event(self.ev_in[s])
        self.s_comp.wait_event(self.ev_out[s])  # O of the call two back has been copied out
        o, _ = self.layers[s].forward(dq, dk, dv, stream=self.s_comp)
        self.ev_comp[s].record(self.s_comp)
        self.s_out.wait_event(self.ev_comp[s])
        with torch.cuda.stream(self.s_out):
            ho.copy_(o, non_blocking=True)
        self.ev_out[s].record(self.s_out)

    def synchronize(self):
        self.s_out.synchronize()
        self.s_comp.synchronize()
        self.s_in.synchronize()


class SubsampledGlobalAttention:
    """Subsampled global attention (AVGGT SGA) for bh heads of S frames x N tokens, N = n_special +
    grid_h * grid_w: keys/values kept on a stride_h x stride_w grid of each frame's patches plus
    every special token, each token's own key, and one mean pair for the other discarded tokens.
    One C call (sa_sga_fwd); the workspace is allocated once."""

    def __init__(self, bh: int, frames: int, tokens: int, grid=(37, 37), stride=(3, 3), n_special: int = 5,
                 dtype: str = "bf16", head_dim: int = 64, device=None, with_lse: bool = True):
        import torch
        self.shape = sa.shape(bh, frames, tokens, head_dim, 128, n_special, dtype)
        self.grid = (int(grid[0]), int(grid[1]))
        self.stride = (int(stride[0]), int(stride[1]))
        nbytes = sa.sa_sga_workspace_size(self.shape, *self.grid, *self.stride)
        if nbytes == 0:
            raise ValueError("unsupported shape or grid for subsampled global attention")
        dev = torch.device(device if device is not None else "cuda")
        self.bh, self.frames, self.tokens, self.d = bh, frames, tokens, head_dim
        self.L = frames * tokens
        self.device = dev
        self.ws = torch.empty((nbytes,), dtype=torch.uint8, device=dev)
        tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
        self.dtype = tdt
        kh = -(-self.grid[0] // self.stride[0])
        kw = -(-self.grid[1] // self.stride[1])
        self.kept_keys = frames * (n_special + kh * kw)  # compacted key sequence per head
        self.o = torch.empty((bh, self.L, head_dim), dtype=tdt, device=dev)
        self.lse = torch.empty((bh, self.L), dtype=torch.float32, device=dev) if with_lse else None

    def forward(self, q, k, v, stream=None):
        sa.sa_sga_fwd(self.shape, *self.grid, *self.stride, q, k, v, self.ws, self.o, self.lse, stream)
        return self.o, self.lse

    __call__ = forward


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
