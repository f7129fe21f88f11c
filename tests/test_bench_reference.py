"""bench.py's reference arm (the fp64 oracle timed on the host cores) on the CPU: a
short run of the tiny workload returns the base contract's JSON fields, and its
length follows the requested time budget rather than the step count."""
import time

import bench
from causal_attention_fwd_attn_b200 import workloads as wl


class Args:
    workload = wl.WORKLOADS[0].name
    mode = None
    steps = 3
    warmup = 3
    reference_seconds = 1.0


def test_reference_arm_line():
    t = time.perf_counter()
    res = bench.run_reference(Args(), rank=0, world=1)
    elapsed = time.perf_counter() - t
    assert res["impl"] == "reference"
    assert res["metric"] == bench.METRIC and res["unit"] == bench.UNIT
    assert res["steps"] == 3 and res["warmup"] == 3
    assert res["value"] > 0 and res["cpu_baseline"]["value"] == res["value"]
    assert res["cpu_baseline"]["kind"] == "oracle" and res["cpu_baseline"]["cores"] >= 1
    assert res["e2e"] == {"value": res["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}
    w = wl.WORKLOADS[0]
    assert res["config"] == bench.config_of(w, w.mode, w.causal, 1)
    # about 1 s of oracle work in all, plus set-up
    assert elapsed < 20


def test_sampler_runs_one_round_per_thread_and_cycles_through_heads():
    w = wl.WORKLOADS[0]
    s = bench.OracleSampler(w, 0, threads=2)
    v, threads, desc, el = s.sample(0.0)
    # a zero budget: the first round (one head pass per thread) is the sample
    assert v > 0 and threads == 2 and desc.startswith("2 head passes")
    assert s.cursor == 2 % w.BH
    s.run_tasks(3, 1)
    assert s.cursor == (2 + 3) % w.BH


def test_sampler_value_counts_the_head_passes():
    w = wl.WORKLOADS[0]
    s = bench.OracleSampler(w, 0, threads=1)
    v, threads, desc, wall = s.sample(0.0)
    assert v * 1e12 * wall == __import__("pytest").approx(w.flops_total() / w.BH, rel=1e-6)
