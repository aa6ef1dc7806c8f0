"""The benchmark's multi-rank logic on CPU: world size 2 over gloo.

Every rank runs its own independent layer call (its own seed), so the only cross-rank
operations are a barrier and the max-reduction of the timings; these tests drive exactly
those functions of bench.py with per-rank timings that differ, on two processes.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        r, wsz, local = bench.rank_env()
        per_rank_ms = 100.0 + 25.0 * rank   # the slowest rank sets the job time
        bench.dist_barrier()
        m = bench.dist_max(per_rank_ms)
        value = bench.whole_job_rate(21984, wsz, 4, m)
        out.put((r, wsz, local, m, bench.rank_seed(0, r), value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_timing_and_weak_scaling():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == 2 for r in res)
    assert all(r[3] == 125.0 for r in res)            # max over ranks, seen by every rank
    assert res[0][4] != res[1][4]                     # independent problems per rank
    # whole-job rate: 2 ranks x 4 steps x 21984 tokens in the slowest rank's 125 ms
    assert res[0][5] == pytest.approx(2 * 4 * 21984 / 0.125)


def test_rank_seeds_give_independent_inputs():
    import bench
    import synth
    from synth.workloads import TINY
    a = synth.generate(TINY, seed=bench.rank_seed(0, 0), heads=1)
    b = synth.generate(TINY, seed=bench.rank_seed(0, 1), heads=1)
    assert not np.array_equal(a["q"], b["q"])


def test_single_process_reductions_are_identity():
    import bench
    assert bench.dist_max(3.5) == 3.5
    assert bench.whole_job_rate(100, 1, 10, 1000.0) == pytest.approx(1000.0)
