"""The GPU arm's JSON line from given measurements (CPU only): the keys the
benchmark contract names, and the arithmetic of value, roofline and launch count."""
import pytest

import bench
from causal_attention_fwd_attn_b200 import workloads as wl

REQUIRED = ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
            "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
            "roofline", "clocks", "e2e", "gpu_launches"]
AVG = {"fwd": 0.95, "pre": 0.05, "dkdv": 2.4}
PEAKS = {"bf16_tflops": 1646.8, "source": "measured"}


def line(world=1, steps=300, traffic=82807296, subs=None):
    _, w = bench.find_workload(bench.DEFAULT_WORKLOAD)
    max_ms = 3.5 * steps
    return w, bench.ours_line(
        w, w.mode, w.causal, steps, 10, world, max_ms, AVG, {"sm_mhz": 1965, "reasons": []},
        {"value": 300.0, "unit": bench.UNIT, "h2d_bytes_per_step": 1, "d2h_bytes_per_step": 1},
        3, PEAKS, traffic, "lib.so", subs)


def test_headline_is_the_largest_workload_in_its_parity_mode():
    w = max(wl.WORKLOADS, key=lambda x: x.flops_total())
    assert bench.DEFAULT_WORKLOAD == w.name
    assert w.mode == "accuracy"


def test_contract_keys_and_types():
    _, res = line()
    for k in REQUIRED:
        assert k in res, k
    assert res["higher_is_better"] is True and res["scaling"] == "weak"
    assert res["vs_baseline"] is None and res["dtype"] == "bf16"
    assert res["config"]["workload"] == bench.DEFAULT_WORKLOAD
    assert res["config"]["mode"] == "accuracy"
    assert "l2" in res["config"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in res["roofline"], k


def test_value_roofline_and_launches():
    w, res = line()
    assert res["value"] == pytest.approx(w.flops_total() / 3.5e-3 / 1e12, abs=0.01)
    achieved = w.flops_bwd() / (AVG["dkdv"] * 1e-3) / 1e12
    assert res["roofline"]["achieved"] == pytest.approx(achieved, abs=0.05)
    assert res["roofline"]["frac"] == pytest.approx(achieved / 1646.8, abs=1e-4)
    assert res["roofline"]["dominant_by_time"] == "dkdv"
    assert res["gpu_launches"] == 3 * 300
    assert res["ms_per_step"] == pytest.approx(3.5)
    assert res["bwd_ms"] == pytest.approx(AVG["pre"] + AVG["dkdv"])


def test_whole_job_value_counts_every_rank():
    _, one = line(world=1)
    _, two = line(world=2)
    assert two["value"] == pytest.approx(2 * one["value"], abs=0.02)
    assert two["n_gpus"] == 2
    # the percentage of peak stays per GPU
    assert two["pct_of_peak"]["measured_bf16"] == pytest.approx(one["pct_of_peak"]["measured_bf16"])


def test_traffic_is_passed_through_or_null():
    assert line(traffic=None)[1]["roofline"]["traffic"] is None


def test_full_attention_counts_twice_the_causal_flops():
    _, w = bench.find_workload("gpt2small_b8h12t1024d64")
    avg = {"fwd": 0.1, "pre": 0.01, "dkdv": 0.2, "cvt": 0.01}
    causal = bench.sub_result(w, "default", 1, 100, 1, 32.0, avg, {}, PEAKS)
    full = bench.sub_result(w, "default", 0, 100, 1, 32.0, avg, {}, PEAKS)
    assert full["value"] == pytest.approx(2 * causal["value"], rel=1e-3)
    assert causal["value"] == pytest.approx(w.flops_total() / 0.32e-3 / 1e12, rel=1e-3)
    assert full["dkdv_frac"] == pytest.approx(2 * causal["dkdv_frac"], rel=1e-3)


def test_both_arms_print_the_same_config():
    _, w = bench.find_workload(bench.DEFAULT_WORKLOAD)

    class Args:
        workload = bench.DEFAULT_WORKLOAD
        mode = None

    ours = line()[1]["config"]
    assert ours == bench.config_of(w, w.mode, w.causal, 1)


def test_sub_results_cover_every_large_workload_and_full_attention():
    names = {n for n, _, _ in bench.SUB_RESULTS}
    assert names >= {w.name for w in wl.WORKLOADS[1:4]}
    assert any(c == 0 for _, _, c in bench.SUB_RESULTS)
