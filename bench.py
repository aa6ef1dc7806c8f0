#!/usr/bin/env python
"""Benchmark: one sparse global-attention layer call (pool -> score -> select -> attend) per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]
                    [--shard replicas|heads]

The default workload is the largest single-GPU one: 1024 frames x 1374 tokens, 16 heads,
97 % tile sparsity with the top-k scoring streamed (no score matrix in memory), with the dense
attention at the same shape timed as the speedup reference.  The three other bf16 workloads
(16, 128 and 512 frames, the last with landmarks) are timed in the same run and reported under
`per_config`.

Prints ONE JSON line (rank 0).  `value` is whole-job tokens/s on the device with inputs
resident in HBM (CUDA events on the launching stream, L2 flushed before every step, max over
ranks); `e2e` is the same metric through the public API with host-resident pinned inputs,
host->device copies of Q/K/V and the device->host read of O inside every timed step.
`roofline` reports the block-sparse attention kernel against the measured bf16 peak, and
`cpu_baseline` the fp64 CPU oracle, run by one process per host core, on a bounded sample of
the same workload.
With N > 1 (torchrun) every rank runs its own independent layer call by default (a different
seed: heads/batches are independent problems), so per-GPU work is fixed ("scaling": "weak");
with --shard heads the ranks split ONE layer call by heads ("scaling": "strong").  Either way
no collective touches the data path; a barrier and a max-reduction of the timings are the
only cross-rank operations.  The overlapped host pipeline (`e2e`) copies every call's inputs
in and its output out inside the timed region.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import shutil
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from synth.workloads import BY_NAME, VGGT_S16, VGGT_S128, VGGT_S512, VGGT_S1024  # noqa: E402

DEFAULT_WORKLOAD = VGGT_S1024.name
# timed beside the default workload in the same run (device figures only)
SIDE_WORKLOADS = [VGGT_S16.name, VGGT_S128.name, VGGT_S512.name]
METRIC = "sparse global-attn tokens/s and kept-tile TFLOPS as % of B200 bf16 peak"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20
L2_NOTE = ("flushed before every step: 256 MB written, then another 256 MB read, so that no dirty line "
           "of the flush is written back inside the timed region")
ATTN_SOURCES = ["view_recon_b200/csrc/k_attn_tc.cuh", "view_recon_b200/csrc/sa_device.cuh"]
# an attention launch at least this long runs inside a seconds-long step under the power cap:
# its fraction is taken against the sustained peak, shorter ones against the burst peak
SUSTAINED_LAUNCH_MS = 50.0


# ------------------------------------------------------------------------------ rank plumbing

def rank_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws an independent problem (weak scaling over independent layer calls)."""
    return base_seed + 1000 * rank


def shard_plan(mode: str, heads: int, world: int, rank: int, base_seed: int):
    """How one rank's work relates to the job.

    mode "replicas": every rank runs its own independent layer call (its own seed), so the job
    is `world` layer calls and per-GPU work is fixed ("weak" scaling).
    mode "heads": the ranks share one layer call; rank r takes heads [r*H/world, (r+1)*H/world)
    of the same draw.  Heads are independent problems end to end, so no data moves between
    ranks ("strong" scaling).
    Returns (heads on this rank, first head, seed, layer calls this rank contributes).
    """
    if mode == "heads" and world > 1:
        if heads % world:
            raise ValueError("--shard heads needs the head count (%d) divisible by the GPU count (%d)"
                             % (heads, world))
        hl = heads // world
        return hl, rank * hl, base_seed, 1.0 / world
    return heads, 0, rank_seed(base_seed, rank), 1.0


def dist_max(value: float, device=None) -> float:
    """Max of a per-rank scalar over the process group (identity without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def whole_job_rate(units_per_rank_step: float, world: int, steps: int, max_total_ms: float) -> float:
    """Units per second for all ranks together, timed as the slowest rank."""
    return units_per_rank_step * world * steps / (max_total_ms / 1e3)


def run_config(w_job, w_local, world: int, sharded: bool) -> dict:
    """The `config` object of a JSON line (identical for the GPU arm and the reference arm)."""
    return {"workload": w_job.name, "frames": w_job.frames, "tokens_per_frame": w_job.tokens,
            "heads": w_job.heads, "head_dim": w_job.head_dim, "tile": w_job.tile, "n_sink": w_job.n_sink,
            "k": w_job.k, "kept_tiles_per_query_tile": w_job.max_kept, "tile_sparsity": round(w_job.sparsity, 4),
            "landmark": w_job.landmark, "streamed_select": w_job.streamed, "l2": L2_NOTE,
            "parallelism": ("%d heads per GPU, one layer call over %d GPUs" % (w_local.heads, world)) if sharded
            else ("independent layer call per GPU" if world > 1 else "single GPU")}


# ------------------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples during the timed region (SM clock, throttle reasons)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, flag in zip(names, parts[5:9]):
                if flag.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


class L2Flush:
    """Evicts the 126 MB L2 before a timed step: writes a 256 MB buffer, then reads another
    256 MB one, so that the lines left in L2 are clean and the timed kernels pay no write-back
    of the flush's own data."""

    def __init__(self, dev):
        import torch
        self.wr = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.acc = torch.zeros((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.wr.zero_()
        self.acc.copy_(self.rd.sum())


# ------------------------------------------------------------------------------ roofline inputs

def measured_peaks() -> tuple[dict, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def tensor_peak(launch_ms: float):
    """(peak TFLOP/s, description, burst peak) for an attention launch of this duration."""
    peaks, src = measured_peaks()
    burst = float(peaks["bf16_tflops"])
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    if launch_ms >= SUSTAINED_LAUNCH_MS:
        return sustained, "%s bf16 sustained (launches of %.0f ms inside a seconds-long step)" % (src, launch_ms), burst
    return burst, "%s bf16 burst" % src, burst


def attn_source_sha() -> str:
    h = hashlib.sha256()
    for rel in ATTN_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the attention kernel from the committed ncu summary, if it was
    taken on the current kernel source; None otherwise."""
    p = os.path.join(ROOT, "profiles", "attn_tc_%s.md" % workload)
    if not os.path.exists(p):
        return None
    text = open(p).read()
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    m_s = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", text)
    if not m_b or not m_s or m_s.group(1) != attn_source_sha():
        return None
    return float(m_b.group(1))


def attention_work(layer, w):
    """Algorithmic FLOPs of one sparse attention launch (4*d per attended (row, key) pair over real
    tokens: listed tiles' key rows, every sink, landmarks) and the tile-granular count (128 x 128
    per listed tile plus the sink chunks)."""
    import torch
    b = layer.buf
    nt, tpf, T = layer.nt, w.tpf, w.tile
    cnt = b.k_cnt.to(torch.int64)
    sinks = w.frames * w.n_sink
    slots = torch.arange(nt, device=cnt.device) % tpf
    rows = torch.clamp(w.tokens - slots * T, max=T).to(torch.int64)  # query rows per tile
    flops, tiles = 0.0, 0.0
    for h in range(b.kept_idx.shape[0]):  # one head at a time bounds the temporaries
        idx = b.kept_idx[h].to(torch.int64)
        valid = idx >= 0
        kc = torch.where(valid, cnt[idx.clamp(min=0)], torch.zeros_like(idx))
        keys = kc.sum(dim=1) + sinks
        if w.landmark:
            keys = keys + (cnt > 0).sum() - (kc > 0).to(torch.int64).sum(dim=1)
        flops += float((keys * rows).sum().item()) * 4 * w.head_dim
        tiles += float(valid.sum().item())
    sink_chunks = -(-sinks // T)
    lm_chunks = (-(-nt // 128)) if w.landmark else 0
    tiles += float(b.kept_idx.shape[0] * nt * (sink_chunks + lm_chunks))
    tile_flops = tiles * T * T * 4 * w.head_dim
    return flops, tile_flops


def with_frames(w, frames: int):
    """The workload at another frame count with the same budget k (so the same number of items per
    query tile, as long as that many candidates exist), under a name that says so."""
    return w.scaled(name="%s_at%d" % (w.name, frames), frames=frames,
                    window=min(w.window, frames) if w.window else 0)


def dense_flops(w, heads):
    return 4.0 * w.head_dim * heads * float(w.L) * float(w.L)


# ------------------------------------------------------------------------------ CPU oracle sample

_OW = {}  # per worker process: the oracle's inputs for the sampled head


def host_cores() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _oracle_worker_init(path, L, d, frames, tokens, tile, n_sink, k, landmark, scale):
    from oracle import oracle as orc
    arr = lambda name, shape: np.load(os.path.join(path, name + ".npy"), mmap_mode="r")  # noqa: E731
    _OW.update(q=arr("q", None), k=arr("k", None), v=arr("v", None), qb=np.load(os.path.join(path, "qb.npy")),
               kb=np.load(os.path.join(path, "kb.npy")), vb=np.load(os.path.join(path, "vb.npy")),
               cnt=np.load(os.path.join(path, "cnt.npy")), g=orc.Geometry(frames, tokens, tile, n_sink),
               k_sel=k, landmark=landmark, scale=scale)


def _oracle_worker_item(i: int) -> int:
    """Score row, selection and attention of query tile i of the sampled head."""
    from oracle import oracle as orc
    o = _OW
    s_row = o["kb"][0] @ o["qb"][0, i]
    kept = orc.select_row(o["g"], s_row, int(i), o["k_sel"])
    orc.attend_tile(o["g"], o["q"], o["k"], o["v"], 0, int(i), kept, o["scale"], o["landmark"], o["kb"], o["vb"],
                    o["cnt"])
    return 1


def _noop(_):
    return 0


class OracleSampler:
    """The fp64 oracle, as it stands, on a bounded sample of one workload, run by one spawned
    process per host core (BLAS single-threaded in each).

    Set-up (once): head 0's inputs are widened to fp64 and pooled in full by the parent; the
    workers map the widened inputs read-only from a temporary directory.  `sample(budget_s)`
    then runs seeded query tiles of that head (score row, selection, attention) on all
    workers for about `budget_s` seconds.  The time of one whole layer call is extrapolated
    as heads x (pooling time + tiles x measured wall time per tile)."""

    def __init__(self, w, data, seed: int = 0):
        import multiprocessing as mp
        from oracle import oracle as orc
        self.w = w
        self.cores = host_cores()
        g = orc.Geometry(w.frames, w.tokens, w.tile, w.n_sink)
        self.nt = g.nt
        t0 = time.perf_counter()
        Q, K, V = (orc.to_f64(data[x][:1]) for x in ("q", "k", "v"))
        qb, kb, vb, cnt, _, _ = orc.pool(g, Q, K, V if w.landmark else None)
        self.t_pool = time.perf_counter() - t0
        self.dir = tempfile.mkdtemp(prefix="oracle_sample_")
        for name, a in (("q", Q), ("k", K), ("v", V), ("qb", qb), ("kb", kb),
                        ("vb", vb if vb is not None else np.zeros((1, 1, 1))), ("cnt", cnt)):
            np.save(os.path.join(self.dir, name + ".npy"), a)
        del Q, K, V
        env_keys = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")
        saved = {x: os.environ.get(x) for x in env_keys}
        for x in env_keys:
            os.environ[x] = "1"
        try:
            ctx = mp.get_context("spawn")
            self.pool = ctx.Pool(self.cores, initializer=_oracle_worker_init,
                                 initargs=(self.dir, w.L, w.head_dim, w.frames, w.tokens, w.tile, w.n_sink, w.k,
                                           w.landmark, 1.0 / np.sqrt(w.head_dim)))
        finally:
            for x, val in saved.items():
                if val is None:
                    os.environ.pop(x, None)
                else:
                    os.environ[x] = val
        self.pool.map(_noop, range(4 * self.cores))  # every worker started and initialised
        self.rng = np.random.default_rng(seed)

    def sample(self, budget_s: float):
        """Returns (tokens/s of one whole layer call, extrapolated; description; full call seconds).
        Keeps one query tile in flight per worker until the budget is spent, then lets the
        ones in flight finish; the wall time covers all of them."""
        from collections import deque
        order = self.rng.permutation(self.nt).tolist()
        pending = deque()
        done = nxt = 0
        t1 = time.perf_counter()
        while nxt < self.nt or pending:
            while len(pending) < self.cores and nxt < self.nt and time.perf_counter() - t1 <= budget_s:
                pending.append(self.pool.apply_async(_oracle_worker_item, (order[nxt],)))
                nxt += 1
            if not pending:
                break
            done += pending.popleft().get()
        wall = time.perf_counter() - t1
        w = self.w
        t_item = wall / max(1, done)  # wall seconds per query tile with every worker busy
        full_s = w.heads * (self.t_pool + self.nt * t_item)
        desc = ("fp64 numpy oracle on %d processes (one per host core): pooling of head 0 of %d (%.2f s, one "
                "process) + %d of %d query tiles of that head (score row, selection, attention) in %.1f s wall, "
                "extrapolated to %d heads x %d tiles = %.0f s per layer call"
                % (self.cores, w.heads, self.t_pool, done, self.nt, wall, w.heads, self.nt, full_s))
        return w.L / full_s, desc, full_s

    def close(self):
        if self.pool is not None:
            self.pool.terminate()
            self.pool.join()
            self.pool = None
        shutil.rmtree(self.dir, ignore_errors=True)


def oracle_baseline(w, data, budget_s: float, seed: int = 0):
    """One bounded oracle sample: (tokens/s, description, cores)."""
    s = OracleSampler(w, data, seed)
    try:
        v, desc, _ = s.sample(budget_s)
    finally:
        s.close()
    return v, desc, s.cores


# ------------------------------------------------------------------------------ the GPU arm

def _pinned(a, dtype: str):
    import torch
    t = torch.from_numpy(a)
    t = t.view(torch.bfloat16) if dtype == "bf16" else t
    return t.pin_memory()


def time_layer(w, q, k, v, dev, steps: int, warmup: int, flush, clocks=None):
    """Warm up, then time `steps` layer calls stage by stage with CUDA events on the current
    stream (L2 flushed before every call).  Returns (layer, per-step stage ms array [steps][4],
    clock record or None)."""
    import torch
    from view_recon_b200 import sa
    from view_recon_b200.pipeline import SparseGlobalAttention
    layer = SparseGlobalAttention(w.heads, w.frames, w.tokens, w.k, w.tile, w.n_sink, w.dtype, w.landmark,
                                  w.streamed, w.head_dim, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step_events():
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        ev[0].record(stream)
        layer.pool(q, k, v)
        ev[1].record(stream)
        layer.score()
        ev[2].record(stream)
        layer.select()
        ev[3].record(stream)
        layer.attend(q, k, v)
        ev[4].record(stream)
        return ev

    for _ in range(warmup):
        flush()
        step_events()
    torch.cuda.synchronize(dev)
    status = sa.sa_check_device_error()
    if status != 0:
        raise RuntimeError("device error after warm-up: %s" % sa.status_string(status))
    if clocks is not None:
        clocks.start()
        time.sleep(0.3)
    dist_barrier(dev)
    torch.cuda.synchronize(dev)
    evs = []
    for _ in range(steps):
        flush()
        evs.append(step_events())
    torch.cuda.synchronize(dev)
    dist_barrier(dev)
    clk = clocks.stop() if clocks is not None else None
    stage = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(4)] for e in evs])  # ms
    status = sa.sa_check_device_error()
    if status != 0:
        raise RuntimeError("device error in timed region: %s" % sa.status_string(status))
    return layer, stage, clk


def time_graph(layer, q, k, v, dev, steps: int, warmup: int, flush) -> float:
    """Mean ms of one layer call replayed from a CUDA graph (the same launches as the eager call,
    recorded once by `SparseGlobalAttention.capture`), L2 flushed before every replay, CUDA
    events on the replaying stream."""
    import torch
    from view_recon_b200 import sa
    g = layer.capture(q, k, v)
    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        flush()
        g.replay()
    torch.cuda.synchronize(dev)
    dist_barrier(dev)
    evs = []
    for _ in range(steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize(dev)
    dist_barrier(dev)
    status = sa.sa_check_device_error()
    if status != 0:
        raise RuntimeError("device error in graph replays: %s" % sa.status_string(status))
    del g
    return float(np.mean([a.elapsed_time(b) for a, b in evs]))


def time_dense(w, q, k, v, dev, flush, budget_s: float = 20.0):
    """Dense control at the same shape: one untimed call, then as many timed calls as fit the
    budget (at least one, at most ten).  Returns mean ms per call."""
    import torch
    from view_recon_b200.pipeline import DenseAttention
    dense = DenseAttention(w.heads, w.frames, w.tokens, w.dtype, w.head_dim, device=dev)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    dense(q, k, v)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    first_ms = e0.elapsed_time(e1)
    n = int(max(1, min(10, budget_s * 1e3 // max(first_ms, 1e-3))))
    pairs = []
    for _ in range(n):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        dense(q, k, v)
        b.record(stream)
        pairs.append((a, b))
    torch.cuda.synchronize(dev)
    del dense
    return float(np.mean([a.elapsed_time(b) for a, b in pairs])), n


def side_config(wname: str, dev, steps: int, warmup: int, flush) -> dict:
    """Device figures of one more workload timed in the same run (one GPU, 16 heads)."""
    import torch
    import synth
    w = BY_NAME[wname]
    host = synth.generate(w)
    q, k, v = (_pinned(host[x], w.dtype).to(dev) for x in ("q", "k", "v"))
    del host
    layer, stage, _ = time_layer(w, q, k, v, dev, steps, warmup, flush)
    ms_pool, ms_score, ms_select, ms_attn = (float(x) for x in stage.mean(axis=0))
    total = float(stage.sum(axis=1).mean())
    flops, tile_flops = attention_work(layer, w)
    peak, peak_desc, burst = tensor_peak(ms_attn)
    achieved = flops / (ms_attn / 1e3) / 1e12
    graph_ms = time_graph(layer, q, k, v, dev, steps, warmup, flush)
    del layer
    dense_ms, n_dense = time_dense(w, q, k, v, dev, flush, budget_s=6.0)
    out = {"tokens_per_s": w.L / (total / 1e3), "ms_per_call": total, "steps": steps,
           "graph_ms_per_call": graph_ms,
           "stages_ms": {"pool": ms_pool, "score": ms_score, "select": ms_select, "attn": ms_attn},
           "attn_tflops_algorithmic": achieved, "attn_tflops_kept_tiles": tile_flops / (ms_attn / 1e3) / 1e12,
           "frac": achieved / peak, "frac_of_burst": achieved / burst, "peak": peak, "peak_source": peak_desc,
           "pool_gbs": (2 + w.landmark) * w.heads * w.L * w.head_dim * 2 / (ms_pool / 1e3) / 1e9,
           "dense_ms": dense_ms, "dense_calls_timed": n_dense, "speedup_vs_dense": dense_ms / total}
    del q, k, v
    torch.cuda.empty_cache()
    return out


def run_ours(args, w):
    import torch
    import torch.distributed as dist

    import synth
    from view_recon_b200 import sa
    from view_recon_b200.pipeline import HostPipeline, SparseGlobalAttention

    rank, world, local = rank_env()
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    sa.load()

    w_job = w
    heads_local, head0, seed, calls_here = shard_plan(args.shard, w.heads, world, rank, w.seed)
    w = w.scaled(heads=heads_local)
    sharded = args.shard == "heads" and world > 1
    # the CPU baseline's workers are spawned before the timed GPU work (they run afterwards)
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    host = synth.generate(w, seed=seed, head0=head0)
    sampler = OracleSampler(w, host) if want_cpu else None
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    hq, hk, hv = (_pinned(host[x], w.dtype) for x in ("q", "k", "v"))
    del host
    q, k, v = hq.to(dev), hk.to(dev), hv.to(dev)
    flush = L2Flush(dev)

    layer, stage, clk = time_layer(w, q, k, v, dev, args.steps, args.warmup, flush, ClockSampler(dev.index))
    total_ms = float(stage.sum())
    max_total_ms = dist_max(total_ms, dev)
    ms_pool, ms_score, ms_select, ms_attn = (float(x) for x in stage.mean(axis=0))
    flops, tile_flops = attention_work(layer, w)
    per_step = layer.launches_per_call()
    max_kept = layer.max_kept
    # the same call replayed from one CUDA graph
    graph_ms = dist_max(time_graph(layer, q, k, v, dev, args.steps, args.warmup, flush), dev)
    del layer
    torch.cuda.empty_cache()

    # dense control at the same shape (speedup reference)
    dense_ms, n_dense = time_dense(w, q, k, v, dev, flush, budget_s=args.dense_budget)

    # end to end through the public API from pinned host buffers: every call copies its Q/K/V in
    # and its O out; HostPipeline overlaps call i's kernels with the copies of calls i+1 and i-1
    del q, k, v
    torch.cuda.empty_cache()
    ho = torch.empty((w.heads, w.L, w.head_dim), dtype=tdt).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    pipe = HostPipeline(lambda: SparseGlobalAttention(w.heads, w.frames, w.tokens, w.k, w.tile, w.n_sink, w.dtype,
                                                      w.landmark, w.streamed, w.head_dim, device=dev))
    for _ in range(2):
        pipe.submit(hq, hk, hv, ho)
    pipe.synchronize()
    torch.cuda.synchronize(dev)
    dist_barrier(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(pipe.s_in)
    for _ in range(e2e_steps):
        pipe.submit(hq, hk, hv, ho)
    e1.record(pipe.s_out)
    torch.cuda.synchronize(dev)
    e2e_ms = dist_max(e0.elapsed_time(e1), dev)
    if sa.sa_check_device_error() != 0:
        raise RuntimeError("device error in the end-to-end leg")
    del pipe
    torch.cuda.empty_cache()
    elem = 2 if w.dtype == "bf16" else 4
    h2d = 3 * w.heads * w.L * w.head_dim * elem
    d2h = w.heads * w.L * w.head_dim * elem

    peak, peak_desc, burst = tensor_peak(ms_attn)
    achieved = flops / (ms_attn / 1e3) / 1e12
    traffic = profiled_traffic(w.name)
    value = whole_job_rate(w.L * calls_here, world, args.steps, max_total_ms)
    line = {
        "metric": METRIC,
        "value": value,
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": max_total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "strong" if sharded else "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic latent-point Q/K/V (seeded; no dataset or weights)",
        "config": run_config(w_job, w, world, sharded),
        "stages_ms": {"pool": ms_pool, "score": ms_score, "select": ms_select, "attn": ms_attn},
        "graph": {"ms_per_call": graph_ms, "tokens_per_s": whole_job_rate(w.L * calls_here, world, 1, graph_ms),
                  "note": "the same call replayed from one CUDA graph (capture once, replay per step)"},
        "attn_tflops_algorithmic": achieved,
        "attn_tflops_kept_tiles": tile_flops / (ms_attn / 1e3) / 1e12,
        "attn_only_tokens_per_s": w.L / (ms_attn / 1e3),
        "pool_gbs": (2 + w.landmark) * w.heads * w.L * w.head_dim * elem / (ms_pool / 1e3) / 1e9,
        "dense_ms": dense_ms,
        "dense_calls_timed": n_dense,
        "dense_tflops": dense_flops(w, w.heads) / (dense_ms / 1e3) / 1e12,
        "speedup_vs_dense": dense_ms / (max_total_ms / args.steps),
        "speedup_vs_dense_attn_only": dense_ms / ms_attn,
        "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel", "achieved": achieved,
                     "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak, "frac_of_burst": achieved / burst,
                     "peak_source": peak_desc,
                     "traffic": traffic,
                     "algorithmic_flops_per_launch": flops,
                     "timed": "attend stage (V^T tile preparation + attention kernel), CUDA events"},
        "e2e": {"value": whole_job_rate(w.L * calls_here, world, e2e_steps, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": per_step * args.steps,
        "clocks": clk,
    }
    assert max_kept == w.max_kept
    if world == 1 and not args.no_side:
        side_steps = max(3, min(args.steps, 10))
        line["per_config"] = {name: side_config(name, dev, side_steps, 3, flush)
                              for name in SIDE_WORKLOADS if name != w.name}
    if sampler is not None:
        try:
            v_cpu, desc, _ = sampler.sample(args.cpu_budget)
        finally:
            sampler.close()
        line["cpu_baseline"] = {"value": v_cpu, "unit": UNIT, "cores": sampler.cores, "kind": "oracle",
                                "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ------------------------------------------------------------------------------ SGA arm

def run_sga(args, w):
    """--sga S: the AVGGT subsampled global attention layer (stride S x S on the 37 x 37 patch grid
    of every frame) on the workload's shape, through the same timing contract."""
    import torch
    import torch.distributed as dist

    import synth
    from view_recon_b200 import sa
    from view_recon_b200.pipeline import HostPipeline, SubsampledGlobalAttention

    rank, world, local = rank_env()
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    sa.load()
    grid = int(round((w.tokens - w.n_sink) ** 0.5))
    if grid * grid + w.n_sink != w.tokens:
        raise SystemExit("--sga needs tokens = n_sink + g * g")
    stride = int(args.sga)
    w_job = w
    heads_local, head0, seed, calls_here = shard_plan(args.shard, w.heads, world, rank, w.seed)
    w = w.scaled(heads=heads_local)
    host = synth.generate(w, seed=seed, head0=head0)

    def pinned(a):
        return torch.from_numpy(a).view(torch.bfloat16).pin_memory()

    hq, hk, hv = pinned(host["q"]), pinned(host["k"]), pinned(host["v"])
    q, k, v = hq.to(dev), hk.to(dev), hv.to(dev)
    make = lambda: SubsampledGlobalAttention(w.heads, w.frames, w.tokens, (grid, grid), (stride, stride),  # noqa: E731
                                             w.n_sink, w.dtype, w.head_dim, device=dev)
    layer = make()
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        flush()
        layer.forward(q, k, v)
    torch.cuda.synchronize(dev)
    if sa.sa_check_device_error() != 0:
        raise RuntimeError("device error after warm-up")
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    dist_barrier(dev)
    torch.cuda.synchronize(dev)
    evs = []
    for _ in range(args.steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        layer.forward(q, k, v)
        e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize(dev)
    dist_barrier(dev)
    clk = clocks.stop()
    total_ms = float(sum(a.elapsed_time(b) for a, b in evs))
    max_total_ms = dist_max(total_ms, dev)
    ms = total_ms / args.steps
    # end to end from pinned host buffers
    ho = torch.empty_like(hq).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    pipe = HostPipeline(make)
    for _ in range(2):
        pipe.submit(hq, hk, hv, ho)
    pipe.synchronize()
    dist_barrier(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(pipe.s_in)
    for _ in range(e2e_steps):
        pipe.submit(hq, hk, hv, ho)
    e1.record(pipe.s_out)
    torch.cuda.synchronize(dev)
    e2e_ms = dist_max(e0.elapsed_time(e1), dev)
    del pipe
    # algorithmic work: every query row over the compacted keys, its diagonal and the mean pair
    flops = 4.0 * w.head_dim * w.heads * float(w.L) * float(layer.kept_keys + 2)
    peak, peak_desc, burst = tensor_peak(ms)
    achieved = flops / (ms / 1e3) / 1e12
    elem = 2
    sharded = args.shard == "heads" and world > 1
    line = {
        "metric": METRIC, "value": whole_job_rate(w.L * calls_here, world, args.steps, max_total_ms),
        "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": max_total_ms / args.steps, "higher_is_better": True,
        "scaling": "strong" if sharded else "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic latent-point Q/K/V (seeded; no dataset or weights)",
        "config": {"workload": "%s_sga%d" % (w_job.name, stride), "frames": w.frames, "tokens_per_frame": w.tokens,
                   "heads": w_job.heads, "head_dim": w.head_dim, "grid": [grid, grid], "stride": [stride, stride],
                   "n_special": w.n_sink, "kept_keys_per_head": layer.kept_keys,
                   "l2": L2_NOTE,
                   "parallelism": ("%d heads per GPU, one layer call over %d GPUs" % (w.heads, world)) if sharded
                   else ("independent layer call per GPU" if world > 1 else "single GPU")},
        "stages_ms": {"sga": ms},
        "attn_tflops_algorithmic": achieved,
        "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel (dense over the kept keys)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "frac_of_burst": achieved / burst, "peak_source": peak_desc,
                     "traffic": None, "algorithmic_flops_per_launch": flops},
        "e2e": {"value": whole_job_rate(w.L * calls_here, world, e2e_steps, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": 3 * w.heads * w.L * w.head_dim * elem,
                "d2h_bytes_per_step": w.heads * w.L * w.head_dim * elem},
        "gpu_launches": 5 * args.steps,  # gather, sums, V^T tiles, attention, combine
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ------------------------------------------------------------------------------ backward arm

def run_backward(args, w):
    """--backward: one training step of the sparse layer, forward (pool, score, select, attend)
    then backward (sa_sparse_attn_bwd) against a fixed upstream gradient, through the same
    timing contract; the roofline is the backward call's (all of its launches)."""
    import torch
    import torch.distributed as dist

    import synth
    from view_recon_b200 import sa
    from view_recon_b200.pipeline import SparseGlobalAttention

    rank, world, local = rank_env()
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    sa.load()
    w_job = w
    heads_local, head0, seed, calls_here = shard_plan(args.shard, w.heads, world, rank, w.seed)
    w = w.scaled(heads=heads_local)
    host = synth.generate(w, seed=seed, head0=head0)

    def pinned(a):
        return torch.from_numpy(a).view(torch.bfloat16).pin_memory()

    rng = np.random.default_rng(seed + 17)
    g32 = rng.standard_normal((w.heads, w.L, w.head_dim)).astype(np.float32)
    gb = g32.view(np.uint32)
    hdo = pinned(((gb + 0x7FFF + ((gb >> 16) & 1)) >> 16).astype(np.uint16))
    hq, hk, hv = pinned(host["q"]), pinned(host["k"]), pinned(host["v"])
    q, k, v, d_o = hq.to(dev), hk.to(dev), hv.to(dev), hdo.to(dev)
    layer = SparseGlobalAttention(w.heads, w.frames, w.tokens, w.k, w.tile, w.n_sink, w.dtype, w.landmark,
                                  w.streamed, w.head_dim, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)

    def step_events():
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(stream)
        layer.forward(q, k, v)
        ev[1].record(stream)
        layer.backward(q, k, v, d_o)
        ev[2].record(stream)
        return ev

    for _ in range(args.warmup):
        flush()
        step_events()
    torch.cuda.synchronize(dev)
    status = sa.sa_check_device_error()
    if status != 0:
        raise RuntimeError("device error after warm-up: %s" % sa.status_string(status))
    fwd_flops, _ = attention_work(layer, w)
    bwd_flops = 2.5 * fwd_flops  # five products of 2*d per attended (row, key) pair against the forward's two
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    dist_barrier(dev)
    torch.cuda.synchronize(dev)
    evs = []
    for _ in range(args.steps):
        flush()
        evs.append(step_events())
    torch.cuda.synchronize(dev)
    dist_barrier(dev)
    clk = clocks.stop()
    st_ms = np.array([[e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2])] for e in evs])
    total_ms = float(st_ms.sum())
    max_total_ms = dist_max(total_ms, dev)
    status = sa.sa_check_device_error()
    if status != 0:
        raise RuntimeError("device error in timed region: %s" % sa.status_string(status))
    ms_fwd, ms_bwd = (float(x) for x in st_ms.mean(axis=0))
    # end to end: Q, K, V and dO in from pinned host memory, dQ, dK, dV out, every step
    hg = [torch.empty_like(hq).pin_memory() for _ in range(3)]
    e2e_steps = max(3, min(args.steps, 10))
    dist_barrier(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        for dst, src in ((q, hq), (k, hk), (v, hv), (d_o, hdo)):
            dst.copy_(src, non_blocking=True)
        layer.forward(q, k, v)
        grads = layer.backward(q, k, v, d_o)
        for dst, src in zip(hg, grads):
            dst.copy_(src, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = dist_max(e0.elapsed_time(e1), dev)
    peak, peak_desc, burst = tensor_peak(ms_bwd)
    achieved = bwd_flops / (ms_bwd / 1e3) / 1e12
    nbytes = w.heads * w.L * w.head_dim * 2
    line = {
        "metric": "sparse global-attention training tokens/s (forward + backward)",
        "value": whole_job_rate(w.L * calls_here, world, args.steps, max_total_ms), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": max_total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak" if not (args.shard == "heads" and world > 1) else "strong",
        "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic latent-point Q/K/V and upstream gradient (seeded; no dataset or weights)",
        "config": {"workload": w_job.name + "_fwd_bwd", "frames": w.frames, "tokens_per_frame": w.tokens,
                   "heads": w_job.heads, "head_dim": w.head_dim, "tile": w.tile, "n_sink": w.n_sink, "k": w.k,
                   "landmark": w.landmark, "l2": L2_NOTE},
        "stages_ms": {"forward": ms_fwd, "backward": ms_bwd},
        "bwd_tflops_algorithmic": achieved,
        "roofline": {"bound": "tensor", "kernel": "sa_sparse_attn_bwd (all launches of the call)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "frac_of_burst": achieved / burst, "peak_source": peak_desc,
                     "traffic": None, "algorithmic_flops_per_launch": bwd_flops},
        "e2e": {"value": whole_job_rate(w.L * calls_here, world, e2e_steps, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": 4 * nbytes, "d2h_bytes_per_step": 3 * nbytes},
        "gpu_launches": (layer.launches_per_call() + layer.backward_launches()) * args.steps,
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del layer
    if world > 1:
        dist.destroy_process_group()


# ------------------------------------------------------------------------------ the reference arm

def run_reference(args, w):
    """The fp64 CPU oracle as the reference arm: every step is a bounded sample of the workload,
    run by one process per host core; under torchrun only rank 0 runs."""
    import synth
    rank, world, _ = rank_env()
    if rank != 0:
        return
    data = synth.generate(w, heads=1)
    sampler = OracleSampler(w, data)
    del data
    vals, descs = [], []
    budget = max(1.0, args.ref_budget / max(1, args.steps + args.warmup))
    try:
        for s in range(args.warmup + args.steps):
            v, desc, _ = sampler.sample(budget)
            if s >= args.warmup:
                vals.append(v)
                descs.append(desc)
    finally:
        sampler.close()
    value = float(np.mean(vals))
    sharded = args.shard == "heads" and world > 1
    w_local = w.scaled(heads=w.heads // world) if sharded else w
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": w.L / value * 1e3,
        "ms_per_step_kind": "extrapolated: one whole layer call, from the timed sample of each step",
        "higher_is_better": True, "scaling": "strong" if sharded else "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic latent-point Q/K/V (seeded; no dataset or weights)",
        "config": run_config(w, w_local, world, sharded),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": sampler.cores, "kind": "oracle",
                         "sample": descs[-1]},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(BY_NAME))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-side", action="store_true", help="skip the per_config timings of the other workloads")
    ap.add_argument("--sga", type=int, default=0, metavar="STRIDE",
                    help="time the AVGGT subsampled global attention layer (stride x stride grid) instead")
    ap.add_argument("--backward", action="store_true",
                    help="time a training step of the sparse layer (forward + backward) instead")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="with N > 1: independent layer call per GPU, or one layer call split by heads")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-budget", type=float, default=90.0, help="seconds of oracle work for --impl reference")
    ap.add_argument("--dense-budget", type=float, default=15.0,
                    help="seconds of timed dense-control calls (at least one call)")
    ap.add_argument("--frames", type=int, default=0,
                    help="run the workload at another frame count, same budget k (smaller profiling cases)")
    ap.add_argument("--heads", type=int, default=0,
                    help="run the workload with fewer heads, same shape per head (smaller profiling cases)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = BY_NAME[args.workload]
    if args.frames:
        w = with_frames(w, args.frames)
    if args.heads:
        w = w.scaled(name="%s_%dheads" % (w.name, args.heads), heads=args.heads)
    if args.impl == "reference":
        run_reference(args, w)
    elif args.sga:
        run_sga(args, w)
    elif args.backward:
        run_backward(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
