"""Benchmark: causal attention forward + backward, bf16, TFLOP/s on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one pass of the whole path over one batch of the workload: the
forward (one kernel) and the backward (D pre-pass, dK/dV kernel with the dQ partials
added by TMA reduce-add into an fp32 accumulator, dQ conversion), all through the C ABI.  FLOPs are the causal counts (forward
2*B*H*T^2*d, backward 2.5x that).  Inputs are synthetic (seeded bf16 Gaussian
with the workload's shape and distribution) and resident in HBM; successive
steps rotate over several input sets whose total is larger than the 126 MB L2.

Prints ONE JSON line on rank 0.  With N > 1 (launched by torch.distributed.run)
every rank runs its own batch (independent heads, no collective on the data
path: weak scaling); the time is the max over ranks.

--impl reference times the fp64 CPU oracle instead (the slow, plain reference
this library is checked against): every step is a bounded sample of whole heads of
the workload, sized so the run takes about --reference-seconds in all (default 150 s
over 3 warm-up and 50 timed steps; a step is never less than one head pass).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from causal_attention_fwd_attn_b200 import workloads as wl  # noqa: E402

METRIC = "causal attention fwd+bwd TFLOP/s (bf16) and % of B200 dense BF16 peak"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "gpt2small_b8h12t1024d64"
L2_BYTES = 126 * 1024 * 1024
PROFILES = os.path.join(ROOT, "profiles")


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"bf16_tflops": p["bf16_tflops"], "bf16_tflops_sustained": p["bf16_tflops_sustained"],
                "hbm_gbs": p["hbm_gbs"], "source": "measured"}
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0,
            "source": "fallback"}


def kernel_source_sha():
    """Hash of the dK/dV kernel's sources (the kernel whose traffic is recorded)."""
    h = hashlib.sha256()
    for name in ("attn_bwd.cu", "sm100_ptx.cuh"):
        with open(os.path.join(ROOT, "causal_attention_fwd_attn_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu capture, if the kernel sources
    are unchanged since it was taken (else None)."""
    path = os.path.join(PROFILES, "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    e = rec.get(kernel, {}).get(workload)
    if not e or e.get("source_sha") != kernel_source_sha():
        return None
    return e.get("dram_bytes_per_launch")


def find_workload(name):
    for i, w in enumerate(wl.WORKLOADS):
        if w.name == name:
            return i, w
    raise SystemExit(f"unknown workload {name}; choose from {[w.name for w in wl.WORKLOADS]}")


class ClockSampler:
    """SM clock, power and clock-event reasons sampled every few milliseconds by an NVML
    thread while the timed region runs.

    mark_begin()/mark_end() bracket the timed region on the host; only samples taken
    between them are reported."""

    REASON_BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40,
                   "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4,
                   "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index, period_s=0.004):
        self.dev = device_index
        self.period = period_s
        self.samples = []  # (host time, sm MHz, power W, reasons bitmask)
        self.handle = None
        self.nvml = None
        self.sm_max = None
        self.thread = None
        self.stop_flag = False
        self.window = [None, None]
        self.error = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = self._handle(pynvml, device_index)
            self.sm_max = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001 - any NVML failure means "no samples"
            self.error = f"nvml unavailable: {type(e).__name__}"
            self.nvml = None

    @staticmethod
    def _handle(pynvml, device_index):
        p = torch.cuda.get_device_properties(device_index)
        bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        return pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())

    def _read(self):
        n = self.nvml
        sm = n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)
        pw = n.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
        rs = n.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
        return sm, pw, rs

    def _loop(self):
        while not self.stop_flag:
            try:
                sm, pw, rs = self._read()
                self.samples.append((time.perf_counter(), sm, pw, rs))
            except Exception as e:  # noqa: BLE001
                self.error = f"nvml read failed: {type(e).__name__}"
                return
            time.sleep(self.period)

    def start(self):
        if self.nvml is None:
            return
        self.thread = threading.Thread(target=self._loop, daemon=True)
        self.thread.start()

    def mark_begin(self):
        self.window[0] = time.perf_counter()

    def mark_end(self):
        self.window[1] = time.perf_counter()

    def stop(self):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=5)
        lo, hi = self.window
        rows = [s for s in self.samples
                if (lo is None or s[0] >= lo) and (hi is None or s[0] <= hi)]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": self.sm_max,
                    "reasons": [self.error or "no samples in the timed region"], "samples": 0}
        reasons = sorted({name for s in rows for name, bit in self.REASON_BITS.items()
                          if s[3] & bit})
        return {"sm_mhz": statistics.median(s[1] for s in rows), "sm_max_mhz": self.sm_max,
                "sm_min_mhz": min(s[1] for s in rows),
                "power_w_median": round(statistics.median(s[2] for s in rows), 1),
                "reasons": reasons, "samples": len(rows), "source": "nvml",
                "period_ms": round(1000 * self.period, 1)}


# ------------------------------------------------------ multi-rank helpers ----
# One process per GPU; every rank runs the whole step on its own batch of heads (the
# heads are independent, so no collective touches the data path).  Only the timing
# is combined: the job is done when its slowest rank is.
def replica_seed_offset(set_index: int, rank: int) -> int:
    """Seed offset of input set `set_index` on `rank` (distinct for fewer than 100
    ranks, since gcd(100, 17) = 1): every rank draws its own heads."""
    return 100 * set_index + 17 * rank


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time, returned on every rank."""
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: each of `world` ranks ran `steps` steps of its own batch
    (weak scaling) within `max_ms`."""
    return flops_per_step * steps * world / (max_ms * 1e-3) / 1e12


# ------------------------------------------------------------------- ours ----
def run_ours(args, rank, world, local_rank):
    from causal_attention_fwd_attn_b200 import _lib

    ci, w = find_workload(args.workload)
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    B, H, T, d = w.B, w.H, w.T, w.d
    scale = w.scale
    set_bytes = 4 * B * H * T * d * 2
    out_bytes = B * H * T * d * 2 * 4 + B * H * T * 4
    n_sets = max(2, math.ceil(3 * L2_BYTES / set_bytes))
    sets = []
    for s in range(n_sets):
        x = wl.make_inputs(ci, seed_offset=replica_seed_offset(s, rank))
        sets.append({n: t.to(dev) for n, t in x.items()})
    o = torch.empty((B, H, T, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty((B, H, T, d), dtype=torch.bfloat16, device=dev) for _ in range(3))
    ws_n = _lib.forge_attn_bwd_workspace_size(B, H, T, d)
    ws = torch.empty(ws_n, dtype=torch.uint8, device=dev)
    rowstats_p = ws.data_ptr()
    acc_p = ws.data_ptr() + _lib.rowstats_bytes(B, H, T)
    stream = torch.cuda.current_stream(dev)
    s = stream.cuda_stream

    def step(x, ev=None):
        q, k, v, dO = x["q"], x["k"], x["v"], x["dO"]
        if ev:
            ev[0].record(stream)
        _lib.check(_lib.forge_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                       lse.data_ptr(), B, H, T, d, scale, w.causal, s), "fwd")
        if ev:
            ev[1].record(stream)
        _lib.check(_lib.forge_attn_bwd_preprocess(o.data_ptr(), dO.data_ptr(), lse.data_ptr(),
                                                  rowstats_p, acc_p, B, H, T, d, 0, s), "pre")
        if ev:
            ev[2].record(stream)
        _lib.check(_lib.forge_attn_bwd_dkdv(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                            dO.data_ptr(), rowstats_p, acc_p, dk.data_ptr(),
                                            dv.data_ptr(), B, H, T, d, scale, w.causal, 0, s),
                   "dkdv")
        if ev:
            ev[3].record(stream)
        _lib.check(_lib.forge_attn_bwd_dq_convert(acc_p, dq.data_ptr(), B, H, T, d, s), "cvt")
        if ev:
            ev[4].record(stream)

    launches_per_step = 4
    for i in range(args.warmup):
        step(sets[i % n_sets])
    torch.cuda.synchronize()
    st, detail = _lib.forge_attn_check_device_error(s)
    if st != _lib.OK:
        raise RuntimeError(f"device wait timed out during warm-up: 0x{detail:08x}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    clocks.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.mark_begin()
    t0.record(stream)
    for i in range(args.steps):
        step(sets[(args.warmup + i) % n_sets], evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    clocks.mark_end()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    elapsed_ms = t0.elapsed_time(t1)
    st, detail = _lib.forge_attn_check_device_error(s)
    if st != _lib.OK:
        raise RuntimeError(f"device wait timed out: 0x{detail:08x}")

    per = {"fwd": [], "pre": [], "dkdv": [], "cvt": []}
    for e in evs:
        per["fwd"].append(e[0].elapsed_time(e[1]))
        per["pre"].append(e[1].elapsed_time(e[2]))
        per["dkdv"].append(e[2].elapsed_time(e[3]))
        per["cvt"].append(e[3].elapsed_time(e[4]))
    avg = {k: sum(v) / len(v) for k, v in per.items()}

    max_ms = max_over_ranks(elapsed_ms, world, dev)

    # ---- end to end through the C ABI with host buffers (pinned) ----------------
    e2e = run_e2e(args, w, ci, dev, stream, o, lse, dq, dk, dv, ws, world)

    if rank != 0:
        return None
    return ours_line(w, args.steps, args.warmup, world, max_ms, avg, clk, e2e,
                     launches_per_step, n_sets, set_bytes, measured_peaks(),
                     recorded_traffic("attn_bwd_dkdv", w.name),
                     os.path.relpath(_lib.library_path(), ROOT))


def ours_line(w, steps, warmup, world, max_ms, avg, clk, e2e, launches_per_step, n_sets,
              set_bytes, peaks, traffic, library):
    """The JSON line of the GPU arm from its measurements: max_ms is the slowest
    rank's time for `steps` steps; avg holds each kernel's mean CUDA-event time (ms)
    per launch ("fwd", "pre", "dkdv", "cvt")."""
    value = job_tflops(w.flops_total(), steps, world, max_ms)
    bwd_ms = avg["pre"] + avg["dkdv"] + avg["cvt"]
    dkdv_flops = w.flops_bwd()
    achieved = dkdv_flops / (avg["dkdv"] * 1e-3) / 1e12
    return {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": steps,
        "warmup": warmup,
        "ms_per_step": round(max_ms / steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": w.name, "B": w.B, "H": w.H, "T": w.T, "d": w.d, "causal": w.causal,
            "scale": "1/sqrt(d)", "inputs": "seeded iid Gaussian bf16, resident in HBM",
            "l2": f"rotating {n_sets} input sets, {n_sets * set_bytes / 2**20:.0f} MiB of "
                  f"inputs > 126 MB L2",
            "parallelism": f"replicas x{world} (independent heads per GPU)",
        },
        "pct_of_peak": {"measured_bf16": round(100 * value / world / peaks["bf16_tflops"], 2),
                        "spec_2250": round(100 * value / world / 2250.0, 2)},
        "fwd_ms": round(avg["fwd"], 4),
        "bwd_ms": round(bwd_ms, 4),
        "kernel_ms": {k: round(v, 4) for k, v in avg.items()},
        "fwd_tflops": round(w.flops_fwd() / (avg["fwd"] * 1e-3) / 1e12, 1),
        "bwd_tflops": round(w.flops_bwd() / (bwd_ms * 1e-3) / 1e12, 1),
        "roofline": {
            "kernel": "attn_bwd_dkdv",
            "bound": "tensor",
            "achieved": round(achieved, 1),
            "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s",
            "frac": round(achieved / peaks["bf16_tflops"], 4),
            "traffic": traffic,
            "peak_source": f"{peaks['source']} bf16_tflops (burst)",
            "dominant_by_time": max(avg, key=avg.get),
            "algorithmic_flops_per_launch": dkdv_flops,
        },
        "clocks": clk,
        "e2e": e2e,
        "gpu_launches": launches_per_step * steps,
        "library": library,
    }


def run_e2e(args, w, ci, dev, stream, o, lse, dq, dk, dv, ws, world):
    """Same metric through the C ABI, with each step's inputs copied from pinned host
    memory and its outputs copied back, all inside the timed region."""
    from causal_attention_fwd_attn_b200 import _lib

    B, H, T, d = w.B, w.H, w.T, w.d
    x = wl.make_inputs(ci, seed_offset=7)
    host_in = {n: t.pin_memory() for n, t in x.items()}
    dev_in = {n: torch.empty_like(t, device=dev) for n, t in x.items()}
    host_out = {"o": torch.empty_like(o, device="cpu").pin_memory(),
                "lse": torch.empty_like(lse, device="cpu").pin_memory(),
                "dq": torch.empty_like(dq, device="cpu").pin_memory(),
                "dk": torch.empty_like(dk, device="cpu").pin_memory(),
                "dv": torch.empty_like(dv, device="cpu").pin_memory()}
    dev_out = {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    s = stream.cuda_stream
    ws_n = ws.numel()

    def step():
        for n in host_in:
            dev_in[n].copy_(host_in[n], non_blocking=True)
        q, k, v, dO = dev_in["q"], dev_in["k"], dev_in["v"], dev_in["dO"]
        _lib.check(_lib.forge_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                       lse.data_ptr(), B, H, T, d, w.scale, w.causal, s), "fwd")
        _lib.check(_lib.forge_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                       dO.data_ptr(), lse.data_ptr(), dq.data_ptr(),
                                       dk.data_ptr(), dv.data_ptr(), ws.data_ptr(), ws_n, B, H,
                                       T, d, w.scale, w.causal, s), "bwd")
        for n in host_out:
            host_out[n].copy_(dev_out[n], non_blocking=True)

    steps = max(3, min(args.steps, 20))
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    value = job_tflops(w.flops_total(), steps, world, ms)
    return {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": round(ms / steps, 4)}


# ---------------------------------------------------------- CPU oracle leg ----
class OracleSampler:
    """Times the fp64 oracle (forward + backward, the full T x T definition) on whole
    heads of a workload, on the host's cores.  The inputs are prepared and the rate
    of head passes with every thread busy is measured once; each sample then runs as
    many head passes as fit its time budget at that rate (at least one), one head per
    thread, cycling through the workload's heads."""

    def __init__(self, w, ci, threads):
        import oracle

        self.w = w
        self.orc = oracle.default()
        x = wl.make_inputs(ci)
        self.f = {n: x[n].double().numpy() for n in x}
        self.heads = [(b, h) for b in range(w.B) for h in range(w.H)]
        self.threads = max(1, threads)
        self.cursor = 0
        nb = min(self.threads, len(self.heads))
        self.rate = nb / max(self._run(self.heads[:nb], nb), 1e-4)  # head passes per second

    def _run(self, hs, threads):
        from concurrent.futures import ThreadPoolExecutor

        f, w, orc = self.f, self.w, self.orc

        def one(bh):
            b, h = bh
            orc.fwd_head(f["q"][b, h], f["k"][b, h], f["v"][b, h], w.scale, w.causal)
            orc.bwd_head(f["q"][b, h], f["k"][b, h], f["v"][b, h], f["dO"][b, h], w.scale,
                         w.causal)

        t = time.perf_counter()
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(one, hs))
        return time.perf_counter() - t

    def sample(self, budget_s):
        """(TFLOP/s in the workload's causal-FLOP convention, threads used,
        description, elapsed seconds) of one sample of about budget_s seconds."""
        w = self.w
        n = max(1, int(budget_s * self.rate))
        threads = min(self.threads, n)
        hs = [self.heads[(self.cursor + j) % len(self.heads)] for j in range(n)]
        self.cursor = (self.cursor + n) % len(self.heads)
        elapsed = self._run(hs, threads)
        value = w.flops_total() / w.BH * n / elapsed / 1e12
        desc = (f"{n} head passes over the {w.BH} heads of {w.name} (T={w.T}, d={w.d}), "
                f"fp64 oracle forward + backward, {elapsed:.2f} s on {threads} threads")
        return value, threads, desc, elapsed


def oracle_sample(w, ci, budget_s, threads):
    """One oracle sample of about budget_s seconds (see OracleSampler)."""
    return OracleSampler(w, ci, threads).sample(budget_s)


def run_reference(args, rank, world):
    """The oracle as it stands, timed on the host cores: each of the warm-up and timed
    steps is one bounded sample of the workload, sized so that the whole run takes
    about args.reference_seconds (a step is never less than one head pass)."""
    if rank != 0:
        return None
    ci, w = find_workload(args.workload)
    sampler = OracleSampler(w, ci, os.cpu_count() or 1)
    budget = args.reference_seconds / max(1, args.steps + args.warmup)
    steps_v, descs, threads = [], [], 1
    for i in range(args.warmup + args.steps):
        v, cores, desc, el = sampler.sample(budget)
        if i >= args.warmup:
            steps_v.append((v, el))
            descs.append(desc)
            threads = max(threads, cores)
    value = statistics.median(v for v, _ in steps_v)
    ms = statistics.median(el for _, el in steps_v) * 1e3
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "T": w.T, "d": w.d,
                   "causal": w.causal, "scale": "1/sqrt(d)",
                   "note": "each step is a bounded sample of the workload's heads"},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": threads,
                         "kind": "oracle", "sample": descs[-1]},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 2000; 50 for --impl reference)")
    ap.add_argument("--warmup", type=int, default=None,
                    help="untimed warm-up steps, at least 3 (default 20; 3 for --impl reference)")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-baseline-seconds", type=float, default=12.0,
                    help="budget of the oracle sample timed beside the GPU run (rank 0, N=1)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--reference-seconds", type=float, default=150.0,
                    help="--impl reference: total oracle time over all warm-up and timed steps "
                         "(each step is at least one head pass)")
    args = ap.parse_args()
    # the reference arm's steps are oracle samples of whole heads (one head pass takes
    # about 0.3 s at the gpt2-small shape on one core), so its default run is shorter
    if args.steps is None:
        args.steps = 50 if args.impl == "reference" else 2000
    if args.warmup is None:
        args.warmup = 3 if args.impl == "reference" else 20
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    if world > 1:
        import datetime

        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=120),
            device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            ci, w = find_workload(args.workload)
            v, cores, desc, _ = oracle_sample(w, ci, args.cpu_baseline_seconds,
                                              os.cpu_count() or 1)
            res["cpu_baseline"] = {"value": round(v, 6), "unit": UNIT, "cores": cores,
                                   "kind": "oracle", "sample": desc}
        elif rank == 0:
            res["cpu_baseline"] = None
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
