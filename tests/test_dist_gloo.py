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


def test_shard_plan_partitions_heads_and_counts_one_call():
    import bench
    for world in (1, 2, 4, 8):
        plans = [bench.shard_plan("heads", 16, world, r, 7) for r in range(world)]
        covered = sorted(h for hl, h0, _, _ in plans for h in range(h0, h0 + hl))
        assert covered == list(range(16))                         # every head exactly once
        assert len({seed for _, _, seed, _ in plans}) == 1        # one draw shared by the ranks
        assert sum(c for *_, c in plans) == pytest.approx(1.0)    # together: one layer call
        reps = [bench.shard_plan("replicas", 16, world, r, 7) for r in range(world)]
        assert all(hl == 16 and h0 == 0 and c == 1.0 for hl, h0, _, c in reps)
        assert len({seed for _, _, seed, _ in reps}) == world     # independent draws
    with pytest.raises(ValueError):
        bench.shard_plan("heads", 16, 3, 0, 7)


def _shard_worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import synth
        from synth.workloads import VGGT_S16
        w = VGGT_S16.scaled(frames=2)
        hl, h0, seed, calls = bench.shard_plan("heads", w.heads, world, rank, w.seed)
        part = synth.generate(w.scaled(heads=hl), seed=seed, head0=h0)
        m = bench.dist_max(50.0 + 10.0 * rank)
        value = bench.whole_job_rate(w.L * calls, world, 3, m)
        out.put((rank, h0, hl, part["q"][:, :64].copy(), value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_head_shards_are_slices_of_one_call():
    import synth
    from synth.workloads import VGGT_S16
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = VGGT_S16.scaled(frames=2)
    full = synth.generate(w)["q"][:, :64]
    for rank, h0, hl, part, value in res:
        assert np.array_equal(part, full[h0:h0 + hl])
        # strong scaling: 3 steps of ONE layer call (w.L tokens) in the slowest rank's 60 ms
        assert value == pytest.approx(3 * w.L / 0.060)
