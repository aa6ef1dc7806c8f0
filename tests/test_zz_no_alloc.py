"""sa_select_topk_noalloc: the selection step for callers that cannot allocate device memory.

Such callers (plugin code inside a framework that owns the device memory pool, or a loop that
must not allocate after start-up) get the streamed selection with the library's own fixed
scratch array instead of a workspace.  Its lists must be exactly those of the workspace-based
call, on two calls in a row with different inputs (the shared array keeps the previous call's
contents, which must not leak into the next result).  This file is collected last so that a
failure here cannot hide any other test.
"""
import ctypes

import numpy as np
import pytest

import synth
from synth.workloads import Workload
from tests import helpers as H

pytestmark = pytest.mark.gpu


def _lists_both_ways(w, seed):
    import torch
    from view_recon_b200 import sa
    lib = sa.load()
    data = synth.generate(w, seed=seed)
    q = H.to_device(data["q"], w.dtype)
    k = H.to_device(data["k"], w.dtype)
    shp = sa.shape_of(w)
    nt = sa.sa_num_tiles(shp)
    mk = sa.sa_max_kept(shp, w.k)
    dev = q.device
    qp = torch.empty((w.heads, nt, 64), dtype=torch.float32, device=dev)
    kp = torch.empty_like(qp)
    cnt = torch.empty((nt,), dtype=torch.int32, device=dev)
    sk = torch.empty((w.heads, max(1, w.frames * w.n_sink), 64), dtype=q.dtype, device=dev)
    sa.sa_tile_pool(shp, q, k, None, qp, kp, None, cnt, sk, None)
    # reference: streamed selection through a caller-provided workspace
    ws = torch.empty((sa.sa_select_workspace_size(shp, True),), dtype=torch.uint8, device=dev)
    idx_ref = torch.full((w.heads, nt, mk), -7, dtype=torch.int32, device=dev)
    cnt_ref = torch.zeros((w.heads, nt), dtype=torch.int32, device=dev)
    sa.sa_select_topk(shp, None, qp, kp, w.k, idx_ref, cnt_ref, mk, ws)
    # the no-allocation entry point, called through the C ABI
    idx = torch.full((w.heads, nt, mk), -7, dtype=torch.int32, device=dev)
    kc = torch.zeros((w.heads, nt), dtype=torch.int32, device=dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.sa_select_topk_noalloc(ctypes.byref(shp), qp.data_ptr(), kp.data_ptr(), w.k, idx.data_ptr(),
                                    kc.data_ptr(), mk, stream)
    assert st == sa.SA_OK, sa.status_string(st)
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0
    return idx.cpu().numpy(), kc.cpu().numpy(), idx_ref.cpu().numpy(), cnt_ref.cpu().numpy()


def test_noalloc_selection_equals_workspace_selection_twice():
    # two calls in a row with different shapes and seeds; lists are integers: compared exactly
    # 140 frames: nt = 1540, more rows than one scratch block holds (1344), so two blocks per head
    first = Workload("noalloc_a", 140, 1374, 2, 64, 128, 5, "bf16", 30, False, True, 2048, 8, 0.7)
    second = Workload("noalloc_b", 9, 700, 2, 64, 128, 5, "bf16", 7, False, True, 256, 0, 0.7)
    for w, seed in ((first, 3), (second, 4)):
        idx, kc, idx_ref, cnt_ref = _lists_both_ways(w, seed)
        assert np.array_equal(kc, cnt_ref)
        assert np.array_equal(idx, idx_ref)
        assert (kc == min(w.k, (w.frames - 1) * w.tpf) + w.tpf).all()


def test_noalloc_rejects_shapes_beyond_its_scratch():
    """The scratch holds 64 rows of the longest row any selection accepts (32768 tiles; a
    static assertion in the library keeps it so), so that row limit is the binding one: a
    longer row is refused before any launch."""
    import torch
    from view_recon_b200 import sa
    lib = sa.load()
    big = sa.shape(1, 3000, 1374, 64, 128, 5, "bf16")  # nt = 33000 > 32768
    dummy = torch.empty((16,), dtype=torch.int32, device="cuda")
    st = lib.sa_select_topk_noalloc(ctypes.byref(big), dummy.data_ptr(), dummy.data_ptr(), 3, dummy.data_ptr(),
                                    dummy.data_ptr(), 1000, None)
    assert st == sa.SA_ERR_UNSUPPORTED
