"""bench.py's reference arm (the fp64 oracle timed on the host cores) on the CPU: a
short run of the tiny workload returns the base contract's JSON fields, and its
length follows the requested time budget rather than the step count."""
import time

import bench
from causal_attention_fwd_attn_b200 import workloads as wl


class Args:
    workload = wl.WORKLOADS[0].name
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
    assert res["config"]["workload"] == Args.workload
    # 1 s of oracle work in all, plus set-up: far below what 6 steps of 2 s would take
    assert elapsed < 20


def test_sampler_runs_at_least_one_head_and_cycles_through_heads():
    w = wl.WORKLOADS[0]
    s = bench.OracleSampler(w, 0, threads=2)
    v, threads, desc, el = s.sample(0.0)
    assert v > 0 and threads == 1 and desc.startswith("1 head passes")
    s.sample(0.0)
    assert s.cursor == 2 % w.BH
