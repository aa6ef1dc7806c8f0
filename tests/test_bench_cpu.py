"""The benchmark's host-side pieces that need no GPU: the reference arm (the fp64 oracle on a
bounded sample, one spawned process per host core) and the choice of the roofline peak."""
import json

import pytest

import bench
from synth.workloads import BY_NAME, TINY, VGGT_S16


def test_reference_arm_line(capsys):
    bench.main(["--impl", "reference", "--workload", TINY.name, "--steps", "3", "--warmup", "3",
                "--ref-budget", "3"])
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    # the same config object as the GPU arm's line for this workload
    assert line["config"] == bench.run_config(TINY, TINY, 1, False)
    assert line["cpu_baseline"]["cores"] == bench.host_cores()
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["value"] > 0 and "extrapolated" in line["ms_per_step_kind"]


def test_oracle_sampler_covers_every_tile_when_the_budget_allows():
    import synth
    w = VGGT_S16.scaled(frames=2, heads=1)
    s = bench.OracleSampler(w, synth.generate(w))
    try:
        v, desc, full_s = s.sample(60.0)
    finally:
        s.close()
    assert "%d of %d query tiles" % (w.nt, w.nt) in desc
    assert v == pytest.approx(w.L / full_s)


def test_peak_choice_by_launch_length():
    peaks, _ = bench.measured_peaks()
    p_short, d_short, burst = bench.tensor_peak(1.0)
    p_long, d_long, _ = bench.tensor_peak(400.0)
    assert p_short == burst == peaks["bf16_tflops"] and "burst" in d_short
    assert p_long == peaks["bf16_tflops_sustained"] and "sustained" in d_long


def test_default_workload_is_the_largest():
    w = BY_NAME[bench.DEFAULT_WORKLOAD]
    assert w.L == max(x.L for x in BY_NAME.values())
    assert w.streamed and bench.DEFAULT_WORKLOAD not in bench.SIDE_WORKLOADS
