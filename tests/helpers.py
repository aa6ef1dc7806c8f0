"""Shared helpers for the GPU parity tests: inputs on the device, outputs back as float64."""
from __future__ import annotations

import numpy as np

import synth
from oracle import oracle as orc


def to_device(arr: np.ndarray, dtype: str):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(arr))
    if dtype == "bf16":
        t = t.view(torch.bfloat16)
    return t.cuda()


def from_device(t) -> np.ndarray:
    """Exact float64 copy of a CUDA tensor (bf16/f32/int)."""
    import torch
    c = t.detach().cpu()
    if c.dtype == torch.bfloat16:
        return orc.to_f64(c.view(torch.int16).numpy().view(np.uint16))
    if c.dtype in (torch.float32, torch.float64):
        return c.numpy().astype(np.float64)
    return c.numpy()


def geometry(w) -> orc.Geometry:
    return orc.Geometry(w.frames, w.tokens, w.tile, w.n_sink)


def inputs(w, heads=None, seed=None):
    d = synth.generate(w, heads=heads, seed=seed)
    return d


def run_gpu(w, data, heads=None, with_lse=True):
    """Run the four-step layer call on the GPU; returns the pipeline object (buffers on device)."""
    from view_recon_b200.pipeline import SparseGlobalAttention
    bh = heads if heads is not None else w.heads
    q = to_device(data["q"], w.dtype)
    k = to_device(data["k"], w.dtype)
    v = to_device(data["v"], w.dtype)
    layer = SparseGlobalAttention(bh, w.frames, w.tokens, w.k, w.tile, w.n_sink, w.dtype, w.landmark,
                                  w.streamed, w.head_dim, with_lse=with_lse)
    layer.forward(q, k, v)
    return layer, (q, k, v)


def kept_lists(layer) -> list:
    idx = from_device(layer.buf.kept_idx)
    cnt = from_device(layer.buf.kept_cnt)
    return [[idx[h, i, : cnt[h, i]].astype(np.int64) for i in range(idx.shape[1])] for h in range(idx.shape[0])]


def check_attention(O_gpu, LSE_gpu, O_ref, LSE_ref, rows_mask=None, max_abs=2e-2, mean_abs=2e-3, lse_abs=1e-2):
    """The output bar: max-abs <= 2e-2 and mean-abs <= 2e-3 over compared elements; LSE abs <= 1e-2."""
    if rows_mask is not None:
        O_gpu, O_ref = O_gpu[rows_mask], O_ref[rows_mask]
        if LSE_gpu is not None:
            LSE_gpu, LSE_ref = LSE_gpu[rows_mask], LSE_ref[rows_mask]
    err = np.abs(O_gpu - O_ref)
    assert np.isfinite(O_gpu).all(), "non-finite GPU output"
    assert err.max() <= max_abs, "max-abs %.3g > %.3g" % (err.max(), max_abs)
    assert err.mean() <= mean_abs, "mean-abs %.3g > %.3g" % (err.mean(), mean_abs)
    if LSE_gpu is not None:
        le = np.abs(LSE_gpu - LSE_ref)
        assert le.max() <= lse_abs, "LSE max-abs %.3g > %.3g" % (le.max(), lse_abs)
    return float(err.max()), float(err.mean())
