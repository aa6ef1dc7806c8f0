"""Thin Python binding of libsa.so (include/sa.h): argument marshalling only.

Every function takes torch CUDA tensors (or None for optional arguments),
checks that they are contiguous and on the current device, and passes raw
pointers and the current stream to the C entry point of the same name.  No
step of the attention path runs in Python, and there is no CPU fallback: if
libsa.so cannot be loaded every call raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsa.so")

SA_OK = 0
SA_ERR_INVALID_ARG = 1
SA_ERR_UNSUPPORTED = 2
SA_ERR_CUDA = 3
SA_ERR_TIMEOUT = 4
SA_ERR_BAD_LIST = 5
SA_ERR_WORKSPACE = 6

SA_F32 = 0
SA_BF16 = 1

# every symbol include/sa.h declares
EXPORTS = [
    "sa_num_tiles", "sa_max_kept", "sa_tile_pool", "sa_tile_scores", "sa_select_workspace_size",
    "sa_select_topk", "sa_select_topk_per_head", "sa_select_topk_noalloc", "sa_head_budget_workspace_size",
    "sa_head_budgets", "sa_sparse_attn_workspace_size", "sa_sparse_attn_fwd", "sa_dense_attn_workspace_size",
    "sa_dense_attn_fwd", "sa_sga_workspace_size", "sa_sga_fwd", "sa_sparse_attn_bwd_workspace_size",
    "sa_sparse_attn_bwd",
    "sa_status_string", "sa_check_device_error", "sa_set_wait_limit_ns", "sa_test_withhold_query_load",
]


class SaShape(ctypes.Structure):
    _fields_ = [
        ("bh", ctypes.c_int32),
        ("frames", ctypes.c_int32),
        ("tokens", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("tile", ctypes.c_int32),
        ("n_sink", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
    ]


class SaError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__("%s failed: %s (status %d)" % (fn, text, status))
        self.status = status


_lib = None


def load(path: str | None = None):
    """Load libsa.so (raises OSError if it is missing: there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise OSError("libsa.so not built at %s (run __graft_entry__.build())" % p)
    lib = ctypes.CDLL(p)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    shp = ctypes.POINTER(SaShape)
    sig = {
        "sa_num_tiles": (i32, [shp]),
        "sa_max_kept": (i32, [shp, i32]),
        "sa_tile_pool": (i32, [shp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]),
        "sa_tile_scores": (i32, [shp, vp, vp, vp, vp]),
        "sa_select_workspace_size": (sz, [shp, i32]),
        "sa_select_topk": (i32, [shp, vp, vp, vp, i32, vp, vp, i32, vp, sz, vp]),
        "sa_select_topk_per_head": (i32, [shp, vp, vp, vp, vp, i32, vp, vp, i32, vp, sz, vp]),
        "sa_select_topk_noalloc": (i32, [shp, vp, vp, i32, vp, vp, i32, vp]),
        "sa_head_budget_workspace_size": (sz, [shp]),
        "sa_head_budgets": (i32, [shp, vp, vp, ctypes.c_float, ctypes.c_float, i32, i32, vp, vp, vp, sz, vp]),
        "sa_sparse_attn_workspace_size": (sz, [shp, i32]),
        "sa_sparse_attn_fwd": (i32, [shp, vp, vp, vp, vp, vp, i32, vp, vp, i32, vp, vp, vp, vp, sz, vp, vp,
                                     vp]),
        "sa_dense_attn_workspace_size": (sz, [shp]),
        "sa_dense_attn_fwd": (i32, [shp, vp, vp, vp, vp, sz, vp, vp, vp]),
        "sa_status_string": (ctypes.c_char_p, [i32]),
        "sa_check_device_error": (i32, [vp]),
        "sa_set_wait_limit_ns": (i32, [ctypes.c_int64]),
        "sa_sga_workspace_size": (sz, [shp, i32, i32, i32, i32]),
        "sa_sga_fwd": (i32, [shp, i32, i32, i32, i32, vp, vp, vp, vp, sz, vp, vp, vp]),
        "sa_test_withhold_query_load": (i32, [i32]),
        "sa_sparse_attn_bwd_workspace_size": (sz, [shp, i32, i32]),
        "sa_sparse_attn_bwd": (i32, [shp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, i32, vp, vp, vp, vp, sz, vp,
                                     vp, vp, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().sa_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != SA_OK:
        raise SaError(fn, status, status_string(status))


def shape(bh, frames, tokens, head_dim=64, tile=128, n_sink=0, dtype="bf16", softmax_scale=0.0) -> SaShape:
    dt = {"bf16": SA_BF16, "f32": SA_F32}[dtype] if isinstance(dtype, str) else int(dtype)
    return SaShape(int(bh), int(frames), int(tokens), int(head_dim), int(tile), int(n_sink), dt,
                   float(softmax_scale))


def shape_of(workload, heads: int | None = None) -> SaShape:
    """sa_shape of a workload description (fields frames, tokens, heads, head_dim, tile, n_sink, dtype)."""
    return shape(heads if heads is not None else workload.heads, workload.frames, workload.tokens,
                 workload.head_dim, workload.tile, workload.n_sink, workload.dtype)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def sa_num_tiles(shp: SaShape) -> int:
    return load().sa_num_tiles(ctypes.byref(shp))


def sa_max_kept(shp: SaShape, k: int) -> int:
    return load().sa_max_kept(ctypes.byref(shp), int(k))


def sa_tile_pool(shp, q, k, v, q_pool, k_pool, v_pool, k_cnt, sink_k, sink_v, stream=None):
    st = load().sa_tile_pool(ctypes.byref(shp), _ptr(q), _ptr(k), _ptr(v), _ptr(q_pool), _ptr(k_pool),
                             _ptr(v_pool), _ptr(k_cnt), _ptr(sink_k), _ptr(sink_v), _stream(stream))
    _check("sa_tile_pool", st)


def sa_tile_scores(shp, q_pool, k_pool, scores, stream=None):
    st = load().sa_tile_scores(ctypes.byref(shp), _ptr(q_pool), _ptr(k_pool), _ptr(scores), _stream(stream))
    _check("sa_tile_scores", st)


def sa_select_workspace_size(shp, streamed: bool) -> int:
    return int(load().sa_select_workspace_size(ctypes.byref(shp), 1 if streamed else 0))


def sa_select_topk(shp, scores, q_pool, k_pool, k, kept_idx, kept_cnt, max_kept, workspace=None, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load().sa_select_topk(ctypes.byref(shp), _ptr(scores), _ptr(q_pool), _ptr(k_pool), int(k),
                               _ptr(kept_idx), _ptr(kept_cnt), int(max_kept), _ptr(workspace), ws_bytes,
                               _stream(stream))
    _check("sa_select_topk", st)


def sa_select_topk_per_head(shp, scores, q_pool, k_pool, k_per_head, k_max, kept_idx, kept_cnt, max_kept,
                            workspace=None, stream=None):
    """k_per_head: int32 device tensor [bh]."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load().sa_select_topk_per_head(ctypes.byref(shp), _ptr(scores), _ptr(q_pool), _ptr(k_pool),
                                        _ptr(k_per_head), int(k_max), _ptr(kept_idx), _ptr(kept_cnt),
                                        int(max_kept), _ptr(workspace), ws_bytes, _stream(stream))
    _check("sa_select_topk_per_head", st)


def sa_head_budget_workspace_size(shp) -> int:
    return int(load().sa_head_budget_workspace_size(ctypes.byref(shp)))


def sa_head_budgets(shp, q_pool, k_pool, temperature, beta, k_lo, k_hi, k_per_head, perplexity=None,
                    workspace=None, stream=None):
    """k_per_head: int32 device tensor [bh] (written); perplexity: f32 device tensor [bh] or None."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load().sa_head_budgets(ctypes.byref(shp), _ptr(q_pool), _ptr(k_pool), float(temperature), float(beta),
                                int(k_lo), int(k_hi), _ptr(k_per_head), _ptr(perplexity), _ptr(workspace), ws_bytes,
                                _stream(stream))
    _check("sa_head_budgets", st)


def sa_select_topk_noalloc(shp, q_pool, k_pool, k, kept_idx, kept_cnt, max_kept, stream=None):
    st = load().sa_select_topk_noalloc(ctypes.byref(shp), _ptr(q_pool), _ptr(k_pool), int(k), _ptr(kept_idx),
                                       _ptr(kept_cnt), int(max_kept), _stream(stream))
    _check("sa_select_topk_noalloc", st)


def sa_sparse_attn_workspace_size(shp, landmark: bool) -> int:
    return int(load().sa_sparse_attn_workspace_size(ctypes.byref(shp), 1 if landmark else 0))


def sa_sparse_attn_fwd(shp, q, k, v, kept_idx, kept_cnt, max_kept, sink_k, sink_v, landmark, k_pool, v_pool,
                       k_cnt, workspace, o, lse=None, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load().sa_sparse_attn_fwd(ctypes.byref(shp), _ptr(q), _ptr(k), _ptr(v), _ptr(kept_idx), _ptr(kept_cnt),
                                   int(max_kept), _ptr(sink_k), _ptr(sink_v), 1 if landmark else 0,
                                   _ptr(k_pool), _ptr(v_pool), _ptr(k_cnt), _ptr(workspace), ws_bytes, _ptr(o),
                                   _ptr(lse), _stream(stream))
    _check("sa_sparse_attn_fwd", st)


def sa_dense_attn_workspace_size(shp) -> int:
    return int(load().sa_dense_attn_workspace_size(ctypes.byref(shp)))


def sa_dense_attn_fwd(shp, q, k, v, workspace, o, lse=None, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load().sa_dense_attn_fwd(ctypes.byref(shp), _ptr(q), _ptr(k), _ptr(v), _ptr(workspace), ws_bytes, _ptr(o),
                                  _ptr(lse), _stream(stream))
    _check("sa_dense_attn_fwd", st)


def sa_sparse_attn_bwd_workspace_size(shp, max_kept, landmark=False) -> int:
    return int(load().sa_sparse_attn_bwd_workspace_size(ctypes.byref(shp), int(max_kept), 1 if landmark else 0))


def sa_sparse_attn_bwd(shp, q, k, v, o, lse, d_o, kept_idx, kept_cnt, max_kept, sink_k, sink_v, landmark, k_pool,
                       v_pool, k_cnt, workspace, dq, dk, dv, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load().sa_sparse_attn_bwd(ctypes.byref(shp), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(d_o),
                                   _ptr(kept_idx), _ptr(kept_cnt), int(max_kept), _ptr(sink_k), _ptr(sink_v),
                                   1 if landmark else 0, _ptr(k_pool), _ptr(v_pool), _ptr(k_cnt), _ptr(workspace),
                                   ws_bytes, _ptr(dq), _ptr(dk), _ptr(dv), _stream(stream))
    _check("sa_sparse_attn_bwd", st)


def sa_check_device_error(stream=None) -> int:
    return int(load().sa_check_device_error(_stream(stream)))


def sa_set_wait_limit_ns(limit_ns: int):
    _check("sa_set_wait_limit_ns", load().sa_set_wait_limit_ns(int(limit_ns)))


def sa_test_withhold_query_load(enable: bool):
    _check("sa_test_withhold_query_load", load().sa_test_withhold_query_load(1 if enable else 0))


def sa_sga_workspace_size(shp, grid_h, grid_w, s_h, s_w) -> int:
    return int(load().sa_sga_workspace_size(ctypes.byref(shp), int(grid_h), int(grid_w), int(s_h), int(s_w)))


def sa_sga_fwd(shp, grid_h, grid_w, s_h, s_w, q, k, v, workspace, o, lse=None, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load().sa_sga_fwd(ctypes.byref(shp), int(grid_h), int(grid_w), int(s_h), int(s_w), _ptr(q), _ptr(k),
                           _ptr(v), _ptr(workspace), ws_bytes, _ptr(o), _ptr(lse), _stream(stream))
    _check("sa_sga_fwd", st)
