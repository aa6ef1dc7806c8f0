#!/usr/bin/env python
"""Benchmark: one sparse global-attention layer call (pool -> score -> select -> attend) per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]
                    [--shard replicas|heads]

Prints ONE JSON line (rank 0).  `value` is whole-job tokens/s on the device with inputs
resident in HBM (CUDA events on the launching stream, L2 flushed before every step, max over
ranks); `e2e` is the same metric through the public API with host-resident pinned inputs,
host->device copies of Q/K/V and the device->host read of O inside every timed step.
`roofline` reports the block-sparse attention kernel against the measured bf16 peak, and
`cpu_baseline` the fp64 CPU oracle on a bounded sample of the same workload.
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
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from synth.workloads import BY_NAME, VGGT_S16  # noqa: E402

DEFAULT_WORKLOAD = VGGT_S16.name
METRIC = "sparse global-attn tokens/s and kept-tile TFLOPS as % of B200 bf16 peak"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 256 << 20
ATTN_SOURCES = ["view_recon_b200/csrc/k_attn_tc.cuh", "view_recon_b200/csrc/sa_device.cuh"]


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


# ------------------------------------------------------------------------------ roofline inputs

def measured_peaks() -> tuple[dict, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


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
    idx = b.kept_idx.to(torch.int64)
    valid = idx >= 0
    keys_listed = torch.where(valid, cnt[idx.clamp(min=0)], torch.zeros_like(idx)).sum(dim=2)  # [bh][nt]
    n_tiles = valid.sum(dim=2)
    sinks = w.frames * w.n_sink
    if w.landmark:
        lm = (cnt > 0).sum() - torch.where(valid, (cnt[idx.clamp(min=0)] > 0).to(torch.int64),
                                            torch.zeros_like(idx)).sum(dim=2)
    else:
        lm = torch.zeros_like(keys_listed)
    keys = keys_listed + sinks + lm
    slots = torch.arange(nt, device=idx.device) % tpf
    rows = torch.clamp(w.tokens - slots * T, max=T).to(torch.int64)  # query rows per tile
    flops = float((keys * rows[None, :]).sum().item()) * 4 * w.head_dim
    sink_chunks = -(-sinks // T)
    lm_chunks = (-(-nt // 128)) if w.landmark else 0
    tiles = float((n_tiles + sink_chunks + lm_chunks).sum().item())
    tile_flops = tiles * T * T * 4 * w.head_dim
    return flops, tile_flops


def dense_flops(w, heads):
    return 4.0 * w.head_dim * heads * float(w.L) * float(w.L)


# ------------------------------------------------------------------------------ CPU oracle sample

def oracle_sample(w, data, budget_s: float = 12.0, seed: int = 0):
    """Time the fp64 oracle on a bounded sample: full pooling of head 0 plus as many seeded
    (head 0, query tile) items (score row, selection, attention) as fit in `budget_s`.
    Returns (tokens/s extrapolated to the whole layer call, description, threads used)."""
    from oracle import oracle as orc
    try:
        from threadpoolctl import threadpool_info
        threads = sum(int(i.get("num_threads", 1)) for i in threadpool_info() if i.get("user_api") == "blas") or 1
    except Exception:  # pragma: no cover
        threads = 1
    g = orc.Geometry(w.frames, w.tokens, w.tile, w.n_sink)
    t0 = time.perf_counter()
    Q, K, V = (orc.to_f64(data[x][:1]) for x in ("q", "k", "v"))
    qb, kb, vb, cnt, _, _ = orc.pool(g, Q, K, V if w.landmark else None)
    t_pool = time.perf_counter() - t0
    rng = np.random.default_rng(seed)
    order = rng.permutation(g.nt)
    t1 = time.perf_counter()
    done = 0
    scale = 1.0 / np.sqrt(w.head_dim)
    for i in order:
        s_row = kb[0] @ qb[0, i]
        kept = orc.select_row(g, s_row, int(i), w.k)
        orc.attend_tile(g, Q, K, V, 0, int(i), kept, scale, w.landmark, kb, vb, cnt)
        done += 1
        if time.perf_counter() - t1 > budget_s:
            break
    t_item = (time.perf_counter() - t1) / max(1, done)
    full_s = w.heads * (t_pool + g.nt * t_item)
    desc = ("fp64 numpy oracle: pooling of 1 of %d heads (%.2f s) + %d of %d query tiles of that head "
            "(score row, selection, attention; %.3f s each), extrapolated to %d heads x %d tiles = %.0f s"
            % (w.heads, t_pool, done, g.nt, t_item, w.heads, g.nt, full_s))
    return w.L / full_s, desc, threads, full_s


# ------------------------------------------------------------------------------ the GPU arm

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
    host = synth.generate(w, seed=seed, head0=head0)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def pinned(a):
        t = torch.from_numpy(a)
        t = t.view(torch.bfloat16) if w.dtype == "bf16" else t
        return t.pin_memory()

    hq, hk, hv = pinned(host["q"]), pinned(host["k"]), pinned(host["v"])
    q, k, v = hq.to(dev), hk.to(dev), hv.to(dev)
    layer = SparseGlobalAttention(w.heads, w.frames, w.tokens, w.k, w.tile, w.n_sink, w.dtype, w.landmark,
                                  w.streamed, w.head_dim, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
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

    for _ in range(args.warmup):
        flush.zero_()
        step_events()
    torch.cuda.synchronize(dev)
    status = sa.sa_check_device_error()
    if status != 0:
        raise RuntimeError("device error after warm-up: %s" % sa.status_string(status))
    flops, tile_flops = attention_work(layer, w)

    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    dist_barrier(dev)
    torch.cuda.synchronize(dev)
    evs = []
    for _ in range(args.steps):
        flush.zero_()
        evs.append(step_events())
    torch.cuda.synchronize(dev)
    dist_barrier(dev)
    clk = clocks.stop()
    stage = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(4)] for e in evs])  # ms
    total_ms = float(stage.sum())
    max_total_ms = dist_max(total_ms, dev)
    status = sa.sa_check_device_error()
    if status != 0:
        raise RuntimeError("device error in timed region: %s" % sa.status_string(status))
    ms_pool, ms_score, ms_select, ms_attn = (float(x) for x in stage.mean(axis=0))

    # dense control at the same shape (speedup reference)
    from view_recon_b200.pipeline import DenseAttention
    dense = DenseAttention(w.heads, w.frames, w.tokens, w.dtype, w.head_dim, device=dev)
    n_dense = max(3, min(10, args.steps))
    for _ in range(2):
        dense(q, k, v)
    d_ms = []
    for _ in range(n_dense):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        dense(q, k, v)
        e1.record(stream)
        d_ms.append((e0, e1))
    torch.cuda.synchronize(dev)
    dense_ms = float(np.mean([a.elapsed_time(b) for a, b in d_ms]))

    # end to end through the public API from pinned host buffers: every call copies its Q/K/V in
    # and its O out; HostPipeline overlaps call i's kernels with the copies of calls i+1 and i-1
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
    del pipe
    elem = 2 if w.dtype == "bf16" else 4
    h2d = 3 * w.heads * w.L * w.head_dim * elem
    d2h = w.heads * w.L * w.head_dim * elem

    peaks, peak_src = measured_peaks()
    achieved = flops / (ms_attn / 1e3) / 1e12
    traffic = profiled_traffic(w.name)
    per_step = layer.launches_per_call()
    value = whole_job_rate(w.L * calls_here, world, args.steps, max_total_ms)
    sharded = args.shard == "heads" and world > 1
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
        "config": {"workload": w_job.name, "frames": w.frames, "tokens_per_frame": w.tokens, "heads": w_job.heads,
                   "head_dim": w.head_dim, "tile": w.tile, "n_sink": w.n_sink, "k": w.k,
                   "kept_tiles_per_query_tile": layer.max_kept, "tile_sparsity": round(w.sparsity, 4),
                   "landmark": w.landmark, "streamed_select": w.streamed, "l2": "flushed before every step",
                   "parallelism": ("%d heads per GPU, one layer call over %d GPUs" % (w.heads, world)) if sharded
                   else ("independent layer call per GPU" if world > 1 else "single GPU")},
        "stages_ms": {"pool": ms_pool, "score": ms_score, "select": ms_select, "attn": ms_attn},
        "attn_tflops_algorithmic": achieved,
        "attn_tflops_kept_tiles": tile_flops / (ms_attn / 1e3) / 1e12,
        "attn_only_tokens_per_s": w.L / (ms_attn / 1e3),
        "dense_ms": dense_ms,
        "dense_tflops": dense_flops(w, w.heads) / (dense_ms / 1e3) / 1e12,
        "speedup_vs_dense": dense_ms / (max_total_ms / args.steps),
        "speedup_vs_dense_attn_only": dense_ms / ms_attn,
        "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel", "achieved": achieved,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                     "peak_source": "%s bf16 burst" % peak_src,
                     "traffic": (traffic if traffic is None else traffic),
                     "algorithmic_flops_per_launch": flops},
        "e2e": {"value": whole_job_rate(w.L * calls_here, world, e2e_steps, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": per_step * args.steps,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v_cpu, desc, threads, _ = oracle_sample(w, host, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": v_cpu, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del layer
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
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        flush.zero_()
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
        flush.zero_()
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
    peaks, peak_src = measured_peaks()
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
                   "l2": "flushed before every step",
                   "parallelism": ("%d heads per GPU, one layer call over %d GPUs" % (w.heads, world)) if sharded
                   else ("independent layer call per GPU" if world > 1 else "single GPU")},
        "stages_ms": {"sga": ms},
        "attn_tflops_algorithmic": achieved,
        "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel (dense over the kept keys)",
                     "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"], "peak_source": "%s bf16 burst" % peak_src,
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
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
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
        flush.zero_()
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
        flush.zero_()
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
    peaks, peak_src = measured_peaks()
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
                   "landmark": w.landmark, "l2": "flushed before every step"},
        "stages_ms": {"forward": ms_fwd, "backward": ms_bwd},
        "bwd_tflops_algorithmic": achieved,
        "roofline": {"bound": "tensor", "kernel": "sa_sparse_attn_bwd (all launches of the call)",
                     "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"], "peak_source": "%s bf16 burst" % peak_src,
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
    """The fp64 CPU oracle as the reference arm: every step is a bounded sample of the workload."""
    import synth
    rank, world, _ = rank_env()
    if rank != 0:
        return
    data = synth.generate(w, heads=1)
    vals, descs, thr = [], [], 1
    budget = max(1.0, args.ref_budget / max(1, args.steps + args.warmup))
    for s in range(args.warmup + args.steps):
        v, desc, thr, _ = oracle_sample(w, data, budget_s=budget, seed=s)
        if s >= args.warmup:
            vals.append(v)
            descs.append(desc)
    value = float(np.mean(vals))
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": w.L / value * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic latent-point Q/K/V (seeded; no dataset or weights)",
        "config": {"workload": w.name, "frames": w.frames, "tokens_per_frame": w.tokens, "heads": w.heads,
                   "head_dim": w.head_dim, "tile": w.tile, "k": w.k},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle", "sample": descs[-1]},
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
    ap.add_argument("--sga", type=int, default=0, metavar="STRIDE",
                    help="time the AVGGT subsampled global attention layer (stride x stride grid) instead")
    ap.add_argument("--backward", action="store_true",
                    help="time a training step of the sparse layer (forward + backward) instead")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="with N > 1: independent layer call per GPU, or one layer call split by heads")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-budget", type=float, default=90.0, help="seconds of oracle work for --impl reference")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = BY_NAME[args.workload]
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
