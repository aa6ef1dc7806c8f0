"""Failure detection on the GPU without a fault: a bounded device wait that runs out.

A test facility withholds one query-tile load of the tensor-core attention kernel, so one
CTA's MMA warp waits for data that never comes.  With a short wait limit the kernel must end
on its own, report SA_ERR_TIMEOUT through the device error word, and leave the context usable:
the next launch (facility off, default limit) is correct again.
"""
import time

import numpy as np
import pytest

from oracle import oracle as orc
from synth.workloads import Workload
from tests import helpers as H

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_is_reported_and_context_survives():
    import torch
    from view_recon_b200 import sa
    w = Workload("timeout", 3, 600, 2, 64, 128, 5, "bf16", 3, False, False, 256, 0, 0.7)
    data = H.inputs(w)
    layer, (q, k, v) = H.run_gpu(w, data)
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0
    try:
        sa.sa_set_wait_limit_ns(50_000_000)      # 50 ms
        sa.sa_test_withhold_query_load(True)
        t0 = time.time()
        layer.attend(q, k, v)
        status = sa.sa_check_device_error()      # synchronises
        elapsed = time.time() - t0
    finally:
        sa.sa_test_withhold_query_load(False)
        sa.sa_set_wait_limit_ns(2_000_000_000)
    assert status == sa.SA_ERR_TIMEOUT
    assert elapsed < 20.0
    assert sa.sa_check_device_error() == 0       # cleared by the read
    # the context is still usable and the next call is correct
    layer.attend(q, k, v)
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0
    g = H.geometry(w)
    Q, K, V = (orc.to_f64(data[x]) for x in ("q", "k", "v"))
    kept = H.kept_lists(layer)
    O_ref, L_ref = orc.attend(g, Q, K, V, kept, 0.125)
    H.check_attention(H.from_device(layer.buf.o), H.from_device(layer.buf.lse), O_ref, L_ref)


def test_backward_wait_that_runs_out_is_reported_and_context_survives():
    """The same facility on the backward: the dQ kernel's first CTA never receives its query
    tile, its MMA warp's wait runs out, the call ends on its own with SA_ERR_TIMEOUT, and the
    next backward (facility off) matches the oracle."""
    import torch
    from view_recon_b200 import sa
    w = Workload("timeout_bwd", 3, 300, 2, 64, 128, 5, "bf16", 2, False, False, 256, 0, 0.7)
    data = H.inputs(w)
    layer, (q, k, v) = H.run_gpu(w, data)
    rng = np.random.default_rng(3)
    f = rng.standard_normal((w.heads, w.L, 64)).astype(np.float32).view(np.uint32)
    do_h = ((f + 0x7FFF + ((f >> 16) & 1)) >> 16).astype(np.uint16)
    d_o = H.to_device(do_h, "bf16")
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0
    try:
        sa.sa_set_wait_limit_ns(50_000_000)      # 50 ms
        sa.sa_test_withhold_query_load(True)
        t0 = time.time()
        layer.backward(q, k, v, d_o)
        status = sa.sa_check_device_error()      # synchronises
        elapsed = time.time() - t0
    finally:
        sa.sa_test_withhold_query_load(False)
        sa.sa_set_wait_limit_ns(2_000_000_000)
    assert status == sa.SA_ERR_TIMEOUT
    assert elapsed < 20.0
    assert sa.sa_check_device_error() == 0
    dq, dk, dv = layer.backward(q, k, v, d_o)
    torch.cuda.synchronize()
    assert sa.sa_check_device_error() == 0
    g = H.geometry(w)
    Q, K, V = (orc.to_f64(data[x]) for x in ("q", "k", "v"))
    ref = orc.attend_backward(g, Q, K, V, H.kept_lists(layer), orc.to_f64(do_h), 0.125)
    for got, want in zip((dq, dk, dv), ref):
        got = H.from_device(got)
        assert np.abs(got - want).max() <= 2e-2 * np.abs(want).max()
