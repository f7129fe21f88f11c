"""The N > 1 path of bench.py on the CPU: two `gloo` ranks, as torchrun would start
them, each timing its own batch; the job's time is the slowest rank's and the
throughput counts every rank's work (independent heads, weak scaling)."""
import datetime
import json
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from causal_attention_fwd_attn_b200 import workloads as wl


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # the same sequence as the timed region: barrier, local timing, barrier, max
        dist.barrier()
        local_ms = 10.0 + 7.5 * rank  # rank 1 is the slower one
        dist.barrier()
        max_ms = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        value = bench.job_tflops(2.0e12, 4, world, max_ms)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"local_ms": local_ms, "max_ms": max_ms, "value": value}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_the_slowest_time(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert [r["max_ms"] for r in res] == [17.5, 17.5]
    # 2 ranks x 4 steps x 2 TFLOP in 17.5 ms
    for r in res:
        assert r["value"] == pytest.approx(2 * 4 * 2.0 / 17.5e-3)


def test_single_rank_needs_no_process_group():
    assert not dist.is_initialized()
    assert bench.max_over_ranks(3.25, 1, torch.device("cpu")) == 3.25
    assert bench.job_tflops(1.0e12, 10, 1, 1000.0) == pytest.approx(10.0)


def test_every_rank_draws_its_own_heads():
    offsets = {bench.replica_seed_offset(s, r) for s in range(16) for r in range(8)}
    assert len(offsets) == 16 * 8
    a = wl.make_inputs(0, seed_offset=bench.replica_seed_offset(0, 0))
    b = wl.make_inputs(0, seed_offset=bench.replica_seed_offset(0, 1))
    for name in ("q", "k", "v", "dO"):
        assert not torch.equal(a[name], b[name])


def test_reference_arm_runs_on_rank_zero_only():
    class Args:
        workload = bench.DEFAULT_WORKLOAD
        steps = 1
        warmup = 3

    # a non-zero rank returns before any oracle work
    assert bench.run_reference(Args(), rank=1, world=2) is None
