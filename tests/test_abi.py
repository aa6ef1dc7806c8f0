"""The C-ABI library without a GPU: it builds, loads, exports every declared symbol, and its
host-side logic (tile counts, list lengths, argument validation) agrees with the oracle."""
import ctypes
import os
import re

import pytest

from oracle import oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from view_recon_b200 import _build, sa
    _build.build()
    return sa.load()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "sa.h")).read()
    return sorted(set(re.findall(r"^\s*(?:[\w\s\*]+?)\b(sa_\w+)\s*\(", text, re.M)))


def test_header_and_binding_agree():
    from view_recon_b200 import sa
    assert declared_symbols() == sorted(sa.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


@pytest.mark.parametrize("S,N,T,ns,k", [(16, 1374, 128, 5, 35), (4, 256, 64, 0, 4), (3, 7, 2, 2, 1),
                                        (1, 700, 128, 5, 9), (5, 300, 64, 5, 1000), (2, 4, 2, 2, 5)])
def test_tile_counts_and_list_lengths(lib, S, N, T, ns, k):
    from view_recon_b200 import sa
    g = orc.Geometry(S, N, T, ns)
    shp = sa.shape(3, S, N, 64, T, ns, "bf16")
    assert sa.sa_num_tiles(shp) == g.nt
    assert sa.sa_max_kept(shp, k) == orc.max_kept(g, k)


def test_invalid_shapes(lib):
    from view_recon_b200 import sa
    assert sa.sa_num_tiles(sa.shape(0, 2, 10)) == -1
    assert sa.sa_num_tiles(sa.shape(1, 2, 10, n_sink=10)) == -1
    assert sa.sa_max_kept(sa.shape(1, 2, 10), -1) == -1
    assert sa.status_string(sa.SA_ERR_TIMEOUT) == "device wait timed out"


def test_validation_happens_before_any_launch(lib):
    # NULL or misaligned pointers are rejected on the host; no CUDA call is made
    from view_recon_b200 import sa
    shp = sa.shape(2, 4, 300, 64, 128, 5, "bf16")
    s = ctypes.byref(shp)
    P = ctypes.c_void_p
    fake = P(0x10000)
    odd = P(0x10008)
    assert lib.sa_tile_pool(s, None, fake, None, fake, fake, None, fake, fake, None, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_tile_pool(s, odd, fake, None, fake, fake, None, fake, fake, None, None) == sa.SA_ERR_INVALID_ARG
    # sinks present but no sink buffer
    assert lib.sa_tile_pool(s, fake, fake, None, fake, fake, None, fake, None, None, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_tile_scores(s, fake, None, fake, None) == sa.SA_ERR_INVALID_ARG
    # max_kept smaller than the list length the budget needs
    assert lib.sa_select_topk(s, fake, None, None, 3, fake, fake, 2, None, 0, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_select_topk(s, fake, None, None, -1, fake, fake, 20, None, 0, None) == sa.SA_ERR_INVALID_ARG
    # streamed selection without its workspace
    assert lib.sa_select_topk(s, None, fake, fake, 3, fake, fake, 20, None, 0, None) == sa.SA_ERR_WORKSPACE
    # per-head budgets: no budget array, a misaligned one, a negative bound, a list too short for the bound
    assert lib.sa_select_topk_per_head(s, fake, None, None, None, 3, fake, fake, 20, None, 0, None) == sa.SA_ERR_INVALID_ARG
    odd2 = P(0x10002)
    assert lib.sa_select_topk_per_head(s, fake, None, None, odd2, 3, fake, fake, 20, None, 0, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_select_topk_per_head(s, fake, None, None, fake, -1, fake, fake, 20, None, 0, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_select_topk_per_head(s, fake, None, None, fake, 3, fake, fake, 2, None, 0, None) == sa.SA_ERR_INVALID_ARG
    # landmark mode without pools
    assert lib.sa_sparse_attn_fwd(s, fake, fake, fake, fake, fake, 6, fake, fake, 1, None, None, None, None, 0,
                                  fake, None, None) == sa.SA_ERR_INVALID_ARG
    # head_dim other than 64 is not built
    bad = sa.shape(2, 4, 300, 32, 128, 0, "bf16")
    assert lib.sa_dense_attn_fwd(ctypes.byref(bad), fake, fake, fake, None, 0, fake, None, None) == sa.SA_ERR_UNSUPPORTED
    # the tensor-core path needs its workspace (transposed V tiles)
    good = sa.shape(2, 4, 300, 64, 128, 0, "bf16")
    assert lib.sa_dense_attn_fwd(ctypes.byref(good), fake, fake, fake, None, 0, fake, None, None) == sa.SA_ERR_WORKSPACE
    assert lib.sa_sparse_attn_fwd(s, fake, fake, fake, fake, fake, 6, fake, fake, 0, None, None, None, None, 0,
                                  fake, None, None) == sa.SA_ERR_WORKSPACE


def test_workspace_sizes(lib):
    from view_recon_b200 import sa
    shp = sa.shape(16, 1024, 1374, 64, 128, 5, "bf16")
    assert sa.sa_select_workspace_size(shp, False) == 0
    ws = sa.sa_select_workspace_size(shp, True)
    assert 0 < ws <= 64 << 20 and ws % (11264 * 4) == 0  # whole score rows, L2-sized
    shp4 = sa.shape(16, 512, 1374, 64, 128, 5, "bf16")
    vt = 16 * 5632 * 64 * 128 * 2                 # transposed V tiles of every key tile
    sinks = 16 * 20 * 64 * 128 * 2                # 512 frames x 5 sinks = 2560 rows = 20 tiles
    assert sa.sa_sparse_attn_workspace_size(shp4, False) == vt + sinks
    assert sa.sa_sparse_attn_workspace_size(shp4, True) >= vt + sinks + 2 * 16 * 5632 * 64 * 2 + 5632 * 4
    assert sa.sa_dense_attn_workspace_size(shp4) == 16 * (-(-512 * 1374 // 128)) * 64 * 128 * 2
    # the 64-key tensor-core path (f32, or tile 64): transposed V in 64-key items of the input type
    # (f32 also keeps Q, K and the sink keys rounded to tf32)
    f32_t64 = sa.shape(2, 4, 256, 64, 64, 0, "f32")          # nt 16, no sinks
    qk = 2 * (2 * 1024 * 64 * 4)
    assert sa.sa_sparse_attn_workspace_size(f32_t64, False) == 2 * 16 * 64 * 64 * 4 + qk
    lm = 2 * 16 * 64 * 64 * 4 + 2 * 64 * 64 * 4 + 2 * 64 * 64 * 4 + 256   # + keys, values, bias (ntp 64)
    assert sa.sa_sparse_attn_workspace_size(f32_t64, True) == lm + qk
    f32_t128 = sa.shape(1, 3, 300, 64, 128, 5, "f32")       # nt 9, two 64-key items per tile, 15 sinks
    sk = -(-15 * 64 * 4 // 256) * 256
    assert sa.sa_sparse_attn_workspace_size(f32_t128, False) == 9 * 2 * 64 * 64 * 4 + 64 * 64 * 4 + \
        2 * 900 * 64 * 4 + sk
    assert sa.sa_dense_attn_workspace_size(sa.shape(2, 4, 256, 64, 64, 0, "bf16")) == 2 * 16 * 64 * 64 * 2


def test_package_fails_loudly_without_library(tmp_path):
    from view_recon_b200 import sa
    with pytest.raises(OSError):
        sa._lib = None
        sa.load(str(tmp_path / "missing.so"))
    sa._lib = None


def test_sga_host_checks(lib):
    from view_recon_b200 import sa
    fake = ctypes.c_void_p(0x10000)
    shp = sa.shape(2, 4, 5 + 37 * 37, 64, 128, 5, "bf16")
    s = ctypes.byref(shp)
    assert lib.sa_sga_workspace_size(s, 37, 37, 3, 3) > 0
    assert lib.sa_sga_workspace_size(s, 36, 37, 3, 3) == 0        # grid does not match the tokens
    assert lib.sa_sga_workspace_size(s, 37, 37, 0, 3) == 0        # stride < 1
    f32 = sa.shape(2, 4, 5 + 37 * 37, 64, 128, 5, "f32")
    assert lib.sa_sga_workspace_size(ctypes.byref(f32), 37, 37, 3, 3) == 0
    assert lib.sa_sga_fwd(s, 36, 37, 3, 3, fake, fake, fake, fake, 1 << 40, fake, None, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_sga_fwd(s, 37, 37, 3, 3, None, fake, fake, fake, 1 << 40, fake, None, None) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_sga_fwd(s, 37, 37, 3, 3, fake, fake, fake, fake, 16, fake, None, None) == sa.SA_ERR_WORKSPACE
    assert lib.sa_sga_fwd(ctypes.byref(f32), 37, 37, 3, 3, fake, fake, fake, fake, 1 << 40, fake, None,
                          None) == sa.SA_ERR_UNSUPPORTED


def test_backward_host_checks(lib):
    from view_recon_b200 import sa
    s = ctypes.byref(sa.shape(2, 3, 300, 64, 128, 5, "bf16"))
    fake = ctypes.c_void_p(0x10000)
    odd = ctypes.c_void_p(0x10008)
    args = lambda **kw: [kw.get(n, fake) for n in ("q", "k", "v", "o", "lse", "do")]  # noqa: E731
    tail = lambda ws=1 << 40: [fake, fake, 0, None, None, None, fake, ws, fake, fake, fake, None]  # noqa: E731
    need = sa.sa_sparse_attn_bwd_workspace_size(sa.shape(2, 3, 300, 64, 128, 5, "bf16"), 5, False)
    assert need > 0
    assert lib.sa_sparse_attn_bwd(s, *args(lse=None), fake, fake, 5, *tail()) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_sparse_attn_bwd(s, *args(o=odd), fake, fake, 5, *tail()) == sa.SA_ERR_INVALID_ARG
    assert lib.sa_sparse_attn_bwd(s, *args(), fake, fake, 0, *tail()) == sa.SA_ERR_INVALID_ARG  # max_kept
    assert lib.sa_sparse_attn_bwd(s, *args(), fake, fake, 5, *tail(ws=need - 1)) == sa.SA_ERR_WORKSPACE
    # sinks missing while the shape has some
    t = tail()
    t[0] = None
    assert lib.sa_sparse_attn_bwd(s, *args(), fake, fake, 5, *t) == sa.SA_ERR_INVALID_ARG
    # landmark mode without the pools
    t = tail()
    t[2] = 1
    assert lib.sa_sparse_attn_bwd(s, *args(), fake, fake, 5, *t) == sa.SA_ERR_INVALID_ARG
    # f32 or tile 64: no backward
    f32 = sa.shape(2, 3, 300, 64, 128, 5, "f32")
    assert sa.sa_sparse_attn_bwd_workspace_size(f32, 5, False) == 0
    assert lib.sa_sparse_attn_bwd(ctypes.byref(f32), *args(), fake, fake, 5, *tail()) == sa.SA_ERR_UNSUPPORTED
    # the workspace grows with the lists and with landmarks
    shp = sa.shape(16, 16, 1374, 64, 128, 5, "bf16")
    assert sa.sa_sparse_attn_bwd_workspace_size(shp, 46, True) > sa.sa_sparse_attn_bwd_workspace_size(shp, 46, False)
    assert sa.sa_sparse_attn_bwd_workspace_size(shp, 100, False) > sa.sa_sparse_attn_bwd_workspace_size(shp, 46, False)


def test_backward_workspace_layout():
    """The backward's workspace is the documented sum of its parts (each rounded to 256 bytes)."""
    from view_recon_b200 import sa
    a256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    bh, S, N, max_kept = 16, 16, 1374, 46
    nt, L = S * 11, S * N
    M = bh * nt
    tile = 64 * 128 * 2
    sink_tiles = -(-S * 5 // 128)
    chunks_q = -(-nt // 32)

    def expect(landmark):
        ntp = -(-nt // 128) * 128
        lm_chunks = ntp // 128 if landmark else 0
        units_cap = bh * (sink_tiles + lm_chunks) * chunks_q + (M * max_kept) // 32 + M + 1
        parts = [M * 128 * 4, M * 128 * 4, M * tile, M * tile, M * tile, bh * sink_tiles * tile,
                 bh * ntp * 128 if landmark else 0, bh * ntp * 128 if landmark else 0,
                 bh * lm_chunks * tile, bh * lm_chunks * tile, ntp * 4 if landmark else 0,
                 M * (ntp // 32) * 4 if landmark else 0, M * 4, M * 4, M * max_kept * 4, units_cap * 16, 16,
                 bh * L * 64 * 4, bh * L * 64 * 4,
                 bh * ntp * 64 * 4 if landmark else 0, bh * ntp * 64 * 4 if landmark else 0]
        return sum(a256(p) for p in parts)

    shp = sa.shape(bh, S, N, 64, 128, 5, "bf16")
    assert sa.sa_sparse_attn_bwd_workspace_size(shp, max_kept, False) == expect(False)
    assert sa.sa_sparse_attn_bwd_workspace_size(shp, max_kept, True) == expect(True)
    assert sa.sa_sparse_attn_bwd_workspace_size(shp, 0, False) == 0          # max_kept out of range
    assert sa.sa_sparse_attn_bwd_workspace_size(shp, nt + 1, False) == 0


def test_head_budget_validation_happens_before_any_launch(lib):
    from view_recon_b200 import sa
    shp = sa.shape(2, 4, 300, 64, 128, 5, "bf16")
    s = ctypes.byref(shp)
    P = ctypes.c_void_p
    fake, odd2 = P(0x10000), P(0x10002)
    nt = sa.sa_num_tiles(shp)
    assert sa.sa_head_budget_workspace_size(shp) == 2 * nt * 4
    ws = 2 * nt * 4
    f = ctypes.c_float
    ok_args = (f(16.0), f(1.0), 0, 10, fake, None, fake, ws, None)
    assert lib.sa_head_budgets(s, None, fake, *ok_args) == sa.SA_ERR_INVALID_ARG           # no q_pool
    assert lib.sa_head_budgets(s, fake, fake, f(16.0), f(1.0), 0, 10, odd2, None, fake, ws,
                               None) == sa.SA_ERR_INVALID_ARG                            # misaligned budgets
    assert lib.sa_head_budgets(s, fake, fake, f(0.0), f(1.0), 0, 10, fake, None, fake, ws,
                               None) == sa.SA_ERR_INVALID_ARG                            # temperature 0
    assert lib.sa_head_budgets(s, fake, fake, f(16.0), f(-1.0), 0, 10, fake, None, fake, ws,
                               None) == sa.SA_ERR_INVALID_ARG                            # negative beta
    assert lib.sa_head_budgets(s, fake, fake, f(16.0), f(1.0), 5, 4, fake, None, fake, ws,
                               None) == sa.SA_ERR_INVALID_ARG                            # k_lo > k_hi
    assert lib.sa_head_budgets(s, fake, fake, f(16.0), f(1.0), 0, 10, fake, None, fake, ws - 4,
                               None) == sa.SA_ERR_WORKSPACE                              # short workspace
