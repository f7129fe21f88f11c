"""The GPU arm's JSON line from given measurements (CPU only): the keys the
benchmark contract names, and the arithmetic of value, roofline and launch count."""
import pytest

import bench

REQUIRED = ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
            "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
            "roofline", "clocks", "e2e", "gpu_launches"]
AVG = {"fwd": 0.0456, "pre": 0.0123, "dkdv": 0.0710, "cvt": 0.0102}


def line(world=1, steps=2000, traffic=82807296):
    _, w = bench.find_workload(bench.DEFAULT_WORKLOAD)
    max_ms = 0.1418 * steps
    return w, bench.ours_line(
        w, steps, 20, world, max_ms, AVG, {"sm_mhz": 1965, "reasons": []},
        {"value": 22.9, "unit": bench.UNIT, "h2d_bytes_per_step": 1, "d2h_bytes_per_step": 1},
        4, 8, 48 << 20, {"bf16_tflops": 1646.8, "source": "measured"}, traffic, "lib.so")


def test_contract_keys_and_types():
    _, res = line()
    for k in REQUIRED:
        assert k in res, k
    assert res["higher_is_better"] is True and res["scaling"] == "weak"
    assert res["vs_baseline"] is None and res["dtype"] == "bf16"
    assert res["config"]["workload"] == bench.DEFAULT_WORKLOAD
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in res["roofline"], k


def test_value_roofline_and_launches():
    w, res = line()
    assert res["value"] == pytest.approx(w.flops_total() / 0.1418e-3 / 1e12, abs=0.01)
    achieved = w.flops_bwd() / (AVG["dkdv"] * 1e-3) / 1e12
    assert res["roofline"]["achieved"] == pytest.approx(achieved, abs=0.05)
    assert res["roofline"]["frac"] == pytest.approx(achieved / 1646.8, abs=1e-4)
    assert res["roofline"]["dominant_by_time"] == "dkdv"
    assert res["gpu_launches"] == 4 * 2000
    assert res["ms_per_step"] == pytest.approx(0.1418)
    assert res["bwd_ms"] == pytest.approx(AVG["pre"] + AVG["dkdv"] + AVG["cvt"])


def test_whole_job_value_counts_every_rank():
    _, one = line(world=1)
    _, two = line(world=2)
    assert two["value"] == pytest.approx(2 * one["value"], abs=0.02)
    assert two["n_gpus"] == 2
    # the percentage of peak stays per GPU
    assert two["pct_of_peak"]["measured_bf16"] == pytest.approx(one["pct_of_peak"]["measured_bf16"])


def test_traffic_is_passed_through_or_null():
    assert line(traffic=None)[1]["roofline"]["traffic"] is None
