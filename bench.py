"""Benchmark: causal attention forward + backward on B200, TFLOP/s and % of the
dense BF16 tensor peak.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--mode MODE]
                    [--impl ours|reference] [--sub-results all|attention|gemm|adamw|none]
                    [--sub-seconds S] [--no-e2e] [--no-cpu-baseline]

One step is one pass of the whole path over one batch of the workload: the forward
(one kernel) and the backward (the D pre-pass, the dK/dV kernel with the dQ partials
added by TMA reduce-add into an fp32 accumulator, and the dQ conversion when dQ is
bf16), all through the C ABI.  FLOPs are the causal counts (forward 2*B*H*T^2*d,
backward 2.5x that; the extra products of the accuracy mode's hi + lo operand
split are not counted).  Inputs are synthetic (seeded bf16 Gaussian with the
workload's shape and distribution) and resident in HBM; successive steps rotate
over several input sets whose total is larger than the 126 MB L2.

The headline workload is the largest one, B=1 H=32 T=8000 d=128 (ragged T), in the
mode that meets the parity tolerances there (its "accuracy" mode: fp32 outputs, D
from the fp32 O, P and dS split into two bf16 terms).  The same line carries
sub-results for the other workloads and for full (non-causal) attention, each timed
over at least half a second of GPU work.

Prints ONE JSON line on rank 0.  With N > 1 (launched by torch.distributed.run)
every rank runs its own batch (independent heads, no collective on the data path:
weak scaling); the time is the max over ranks.

--impl reference times the fp64 CPU oracle instead (the slow, plain reference this
library is checked against) on the same workload: every step is a bounded sample
of whole heads; the steps run concurrently on the host's cores.
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
DEFAULT_WORKLOAD = "ragged_b1h32t8000d128"
L2_BYTES = 126 * 1024 * 1024
PROFILES = os.path.join(ROOT, "profiles")
# Sub-results beside the headline: (workload, mode, causal).  Every causal workload
# in the mode its parity tests use, the long workload also in the default bf16 mode
# (context: outside the tolerance there) and in the fp16-operand accuracy mode (which
# meets the tolerance there too, with its bf16 -> fp16 input conversion in the step),
# and full attention at two shapes.
SUB_RESULTS = [
    ("gpt2small_b8h12t1024d64", "default", 1),
    ("decoder200m_b4h16t2048d64", "default", 1),
    ("hd128_b2h16t4096d128", "default", 1),
    ("ragged_b1h32t8000d128", "default", 1),
    ("ragged_b1h32t8000d128", "accuracy_fp16", 1),
    ("gpt2small_b8h12t1024d64", "default", 0),
    ("hd128_b2h16t4096d128", "default", 0),
]
SUB_RESULT_SECONDS = 0.5  # default; --sub-seconds


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


def recorded_traffic(kernel, key):
    """DRAM bytes per launch from a committed ncu capture, if the kernel sources
    are unchanged since it was taken (else None)."""
    path = os.path.join(PROFILES, "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    e = rec.get(kernel, {}).get(key)
    if not e or e.get("source_sha") != kernel_source_sha():
        return None
    return e.get("dram_bytes_per_launch")


def find_workload(name):
    try:
        return wl.find(name)
    except KeyError as e:
        raise SystemExit(str(e)) from None


def causal_flops(w, causal):
    """(forward, backward) FLOPs of one pass: the causal counts, twice that for full
    attention."""
    f = 1.0 if causal else 2.0
    return f * w.flops_fwd(), f * w.flops_bwd()


def n_input_sets(w):
    set_bytes = 4 * w.B * w.H * w.T * w.d * 2
    return max(2, math.ceil(3 * L2_BYTES / set_bytes)), set_bytes


def config_of(w, mode, causal, world):
    """The workload description both arms print (identical keys and values)."""
    n_sets, set_bytes = n_input_sets(w)
    return {
        "workload": w.name, "B": w.B, "H": w.H, "T": w.T, "d": w.d, "causal": causal,
        "scale": "1/sqrt(d)", "mode": mode,
        "inputs": "seeded iid Gaussian bf16 (seed 1000*workload + tensor), resident in HBM",
        "l2": f"inputs larger than L2: rotating {n_sets} input sets, "
              f"{n_sets * set_bytes / 2**20:.0f} MiB > 126 MB L2",
        "parallelism": f"replicas x{world} (independent heads per GPU)",
    }


class ClockSampler:
    """SM clock, power and clock-event reasons sampled every few milliseconds by an NVML
    thread.  window_begin()/window_end() bracket a timed region on the host; stats()
    summarises the samples taken inside one window."""

    REASON_BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40,
                   "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4,
                   "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index, period_s=0.002):
        self.dev = device_index
        self.period = period_s
        self.samples = []  # (host time, sm MHz, power W, reasons bitmask)
        self.lock = threading.Lock()
        self.handle = None
        self.nvml = None
        self.sm_max = None
        self.thread = None
        self.stop_flag = False
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
                with self.lock:
                    self.samples.append((time.perf_counter(), sm, pw, rs))
            except Exception as e:  # noqa: BLE001
                self.error = f"nvml read failed: {type(e).__name__}"
                return
            time.sleep(self.period)

    def start(self):
        if self.nvml is not None and self.thread is None:
            self.thread = threading.Thread(target=self._loop, daemon=True)
            self.thread.start()
        return self

    def stop(self):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=5)
            self.thread = None

    @staticmethod
    def now():
        return time.perf_counter()

    def stats(self, lo, hi):
        with self.lock:
            rows = [s for s in self.samples if lo <= s[0] <= hi]
        return summarise_clocks(rows, self.sm_max, self.error, self.period)


def summarise_clocks(rows, sm_max, error=None, period=0.002):
    """Median SM clock, power and the clock-event reasons seen in `rows` of
    (time, sm MHz, power W, reasons bitmask)."""
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": sm_max,
                "reasons": [error or "no samples in the timed region"], "samples": 0}
    reasons = sorted({name for s in rows for name, bit in ClockSampler.REASON_BITS.items()
                      if s[3] & bit})
    return {"sm_mhz": statistics.median(s[1] for s in rows), "sm_max_mhz": sm_max,
            "sm_min_mhz": min(s[1] for s in rows),
            "power_w_median": round(statistics.median(s[2] for s in rows), 1),
            "reasons": reasons, "samples": len(rows), "source": "nvml",
            "period_ms": round(1000 * period, 1)}


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


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


# ------------------------------------------------------------------- ours ----
class Pass:
    """Device buffers and the launches of one step (forward + backward) of a workload
    in a mode, through the C ABI's stage entry points."""

    def __init__(self, w, mode, causal, dev):
        from causal_attention_fwd_attn_b200 import _lib

        self.lib = _lib
        self.w, self.mode, self.causal = w, mode, causal
        m = wl.MODES[mode]
        B, H, T, d = w.B, w.H, w.T, w.d
        odt = torch.float32 if m["o_f32"] else torch.bfloat16
        gdt = torch.float32 if m["grad_f32"] else torch.bfloat16
        self.o = torch.empty((B, H, T, d), dtype=odt, device=dev)
        self.lse = torch.empty((B, H, T), dtype=torch.float32, device=dev)
        self.dq, self.dk, self.dv = (torch.empty((B, H, T, d), dtype=gdt, device=dev)
                                     for _ in range(3))
        self.ws_n = _lib.forge_attn_bwd_workspace_size(B, H, T, d)
        self.ws = torch.empty(self.ws_n, dtype=torch.uint8, device=dev)
        self.rowstats = self.ws.data_ptr()
        # with fp32 gradients the dQ accumulator is dq itself, and there is no conversion
        self.acc = (self.dq.data_ptr() if m["grad_f32"]
                    else self.ws.data_ptr() + _lib.rowstats_bytes(B, H, T))
        # the fp16-operand mode converts each step's bf16 inputs into these first
        self.fp16 = m["fp16"]
        self.x16 = ({n: torch.empty((B, H, T, d), dtype=torch.float16, device=dev)
                     for n in ("q", "k", "v", "dO")} if self.fp16 else None)
        self.overflow = torch.zeros(1, dtype=torch.int32, device=dev)
        p = (_lib.PRECISE if m["precise"] else 0) | (_lib.FP16 if self.fp16 else 0)
        self.fwd_flags = (_lib.OUT_F32 if m["o_f32"] else 0) | p
        self.pre_flags = (_lib.O_IN_F32 if m["o_f32"] else 0) | (_lib.FP16 if self.fp16 else 0)
        self.dkdv_flags = (_lib.OUT_F32 if m["grad_f32"] else 0) | p
        self.bwd_flags = self.pre_flags | self.dkdv_flags
        # timed stages in step order ("in": the four input conversions)
        self.kernels = ((["in"] if self.fp16 else []) + ["fwd", "pre", "dkdv"]
                        + ([] if m["grad_f32"] else ["cvt"]))
        self.launches_per_step = len(self.kernels) + (3 if self.fp16 else 0)
        self.stream = torch.cuda.current_stream(dev)

    def to_fp16(self, x):
        """The library's bf16 -> fp16 conversion of q, k, v, dO into self.x16."""
        L, s = self.lib, self.stream.cuda_stream
        for n in ("q", "k", "v", "dO"):
            L.check(L.forge_attn_bf16_to_fp16(x[n].data_ptr(), self.x16[n].data_ptr(),
                                              x[n].numel(), self.overflow.data_ptr(), s),
                    "bf16_to_fp16")
        return self.x16

    def step(self, x, ev=None):
        """One step; with `ev` (five events) an event before the first stage and after
        each stage of self.kernels."""
        L, w, s = self.lib, self.w, self.stream.cuda_stream
        B, H, T, d = w.B, w.H, w.T, w.d
        marks = iter(ev or [])

        def mark():
            if ev:
                next(marks).record(self.stream)

        mark()
        if self.fp16:
            x = self.to_fp16(x)
            mark()
        q, k, v, dO = x["q"], x["k"], x["v"], x["dO"]
        L.check(L.forge_attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), self.o.data_ptr(),
                                    self.lse.data_ptr(), B, H, T, d, w.scale, self.causal,
                                    self.fwd_flags, s), "fwd")
        mark()
        L.check(L.forge_attn_bwd_preprocess(self.o.data_ptr(), dO.data_ptr(), self.lse.data_ptr(),
                                            self.rowstats, self.acc, B, H, T, d, self.pre_flags,
                                            s), "pre")
        mark()
        L.check(L.forge_attn_bwd_dkdv(q.data_ptr(), k.data_ptr(), v.data_ptr(), dO.data_ptr(),
                                      self.rowstats, self.acc, self.dk.data_ptr(),
                                      self.dv.data_ptr(), B, H, T, d, w.scale, self.causal,
                                      self.dkdv_flags, s), "dkdv")
        mark()
        if "cvt" in self.kernels:
            L.check(L.forge_attn_bwd_dq_convert(self.acc, self.dq.data_ptr(), B, H, T, d, s),
                    "cvt")
            mark()

    def kernel_times(self, evs):
        """Mean CUDA-event time (ms) of each stage over the steps of `evs`."""
        per = {k: [] for k in self.kernels}
        for e in evs:
            for a, k in enumerate(self.kernels):
                per[k].append(e[a].elapsed_time(e[a + 1]))
        return {k: sum(v) / len(v) for k, v in per.items()}

    def check_device(self, when):
        st, detail = self.lib.forge_attn_check_device_error(self.stream.cuda_stream)
        if st != self.lib.OK:
            raise RuntimeError(f"device wait timed out {when}: 0x{detail:08x}")


def input_sets(ci, w, rank, dev):
    n_sets, _ = n_input_sets(w)
    return [{n: t.to(dev) for n, t in
             wl.make_inputs(ci, w, seed_offset=replica_seed_offset(s, rank)).items()}
            for s in range(n_sets)]


def timed_run(p, sets, warmup, steps, world, dev, clocks):
    """`warmup` untimed steps, then exactly `steps` steps between barriers and device
    synchronisations.  Returns (max-over-ranks ms, per-kernel mean ms, clock stats)."""
    n_sets = len(sets)
    for i in range(warmup):
        p.step(sets[i % n_sets])
    torch.cuda.synchronize()
    p.check_device("during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    lo = clocks.now()
    t0.record(p.stream)
    for i in range(steps):
        p.step(sets[(warmup + i) % n_sets], evs[i])
    t1.record(p.stream)
    torch.cuda.synchronize()
    hi = clocks.now()
    barrier(world)
    p.check_device("in the timed region")
    if p.fp16 and int(p.overflow.item()) != 0:
        raise RuntimeError("inputs beyond fp16's range in the fp16-operand mode")
    max_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    return max_ms, p.kernel_times(evs), clocks.stats(lo, hi)


def dominant(avg):
    return max(avg, key=avg.get)


def roofline_of(w, causal, avg, peaks, traffic):
    """Roofline object of the dK/dV kernel (the dominant one): its algorithmic FLOPs
    per launch (the backward's causal count) over its mean CUDA-event duration."""
    _, bwd_flops = causal_flops(w, causal)
    achieved = bwd_flops / (avg["dkdv"] * 1e-3) / 1e12
    return {
        "kernel": "attn_bwd_dkdv",
        "bound": "tensor",
        "achieved": round(achieved, 1),
        "peak": peaks["bf16_tflops"],
        "unit": "TFLOP/s",
        "frac": round(achieved / peaks["bf16_tflops"], 4),
        "traffic": traffic,
        "peak_source": f"{peaks['source']} bf16_tflops (burst)",
        "dominant_by_time": dominant(avg),
        "algorithmic_flops_per_launch": bwd_flops,
    }


def result_fields(w, causal, steps, world, max_ms, avg, peaks):
    """Throughput fields shared by the headline and the sub-results."""
    fwd_flops, bwd_flops = causal_flops(w, causal)
    value = job_tflops(fwd_flops + bwd_flops, steps, world, max_ms)
    bwd_ms = sum(v for k, v in avg.items() if k not in ("fwd", "in"))
    return {
        "value": round(value, 2),
        "ms_per_step": round(max_ms / steps, 4),
        "pct_of_peak": {"measured_bf16" if peaks["source"] == "measured" else "fallback_bf16":
                        round(100 * value / world / peaks["bf16_tflops"], 2),
                        "spec_2250": round(100 * value / world / 2250.0, 2)},
        "fwd_ms": round(avg["fwd"], 4),
        "bwd_ms": round(bwd_ms, 4),
        "kernel_ms": {k: round(v, 4) for k, v in avg.items()},
        "fwd_tflops": round(fwd_flops / (avg["fwd"] * 1e-3) / 1e12, 1),
        "bwd_tflops": round(bwd_flops / (bwd_ms * 1e-3) / 1e12, 1),
    }


def ours_line(w, mode, causal, steps, warmup, world, max_ms, avg, clk, e2e, launches_per_step,
              peaks, traffic, library, sub_results=None):
    """The JSON line of the GPU arm from its measurements: max_ms is the slowest
    rank's time for `steps` steps; avg holds each kernel's mean CUDA-event time (ms)
    per launch ("fwd", "pre", "dkdv" and, with bf16 gradients, "cvt")."""
    r = result_fields(w, causal, steps, world, max_ms, avg, peaks)
    line = {
        "metric": METRIC,
        "value": r.pop("value"),
        "unit": UNIT,
        "n_gpus": world,
        "steps": steps,
        "warmup": warmup,
        "ms_per_step": r.pop("ms_per_step"),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16" if wl.MODES[mode]["fp16"] else "bf16",
        "data": "synthetic",
        "config": config_of(w, mode, causal, world),
        "mode_desc": wl.MODES[mode]["desc"],
    }
    line.update(r)
    line.update({
        "roofline": roofline_of(w, causal, avg, peaks, traffic),
        "clocks": clk,
        "e2e": e2e,
        "gpu_launches": launches_per_step * steps,
        "library": library,
    })
    if sub_results is not None:
        line["sub_results"] = sub_results
    return line


def sub_result(w, mode, causal, steps, world, max_ms, avg, clk, peaks):
    r = result_fields(w, causal, steps, world, max_ms, avg, peaks)
    _, bwd_flops = causal_flops(w, causal)
    dkdv_tf = bwd_flops / (avg["dkdv"] * 1e-3) / 1e12
    r.update({"workload": w.name, "mode": mode, "causal": causal, "steps": steps,
              "dtype": "f16" if wl.MODES[mode]["fp16"] else "bf16",
              "dominant_kernel": dominant(avg),
              "dkdv_frac": round(dkdv_tf / peaks["bf16_tflops"], 4),
              "clocks": {k: clk.get(k) for k in ("sm_mhz", "samples", "reasons")}})
    return r


def run_sub_results(rank, world, dev, clocks, peaks, warmup, seconds):
    """Each (workload, mode, causal) of SUB_RESULTS timed over at least `seconds` of GPU
    work, 20 steps at least (the step count is sized from the warm-up steps and agreed
    over ranks)."""
    out = []
    for name, mode, causal in SUB_RESULTS:
        ci, w = find_workload(name)
        sets = input_sets(ci, w, rank, dev)
        p = Pass(w, mode, causal, dev)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for i in range(warmup):
            p.step(sets[i % len(sets)])
        t0.record(p.stream)
        for i in range(3):
            p.step(sets[i % len(sets)])
        t1.record(p.stream)
        torch.cuda.synchronize()
        est_ms = max_over_ranks(t0.elapsed_time(t1) / 3, world, dev)
        steps = max(20, min(20000, math.ceil(seconds * 1e3 / est_ms)))
        max_ms, avg, clk = timed_run(p, sets, 3, steps, world, dev, clocks)
        out.append(sub_result(w, mode, causal, steps, world, max_ms, avg, clk, peaks))
        del sets, p
        torch.cuda.empty_cache()
    return out


# ------------------------------------------- the other hot-path kernels -------
# The projection GEMMs around attention and the fused AdamW step, each timed over at
# least --sub-seconds with input sets rotating through more than the L2.
GEMM_SUB_RESULTS = [
    # (name, tokens, in_features, out_features, product)
    ("square4096_fwd", 4096, 4096, 4096, "fwd"),
    ("gpt2small_mlp_fc_fwd", 8192, 768, 3072, "fwd"),
    ("gpt2small_mlp_fc_dx", 8192, 768, 3072, "dx"),
    ("gpt2small_mlp_fc_dw", 8192, 768, 3072, "dw"),
]


def gemm_flops(tokens, din, dout):
    return 2.0 * tokens * din * dout


def time_loop(fn, n_sets, world, dev, clocks, seconds, warmup=3):
    """fn(i) launches step i; sizes the timed loop to `seconds` from three
    probe steps (agreed over ranks) and returns (steps, max-over-ranks ms, clock stats)."""
    stream = torch.cuda.current_stream(dev)
    for i in range(warmup):
        fn(i % n_sets)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(3):
        fn(i % n_sets)
    t1.record(stream)
    torch.cuda.synchronize()
    est = max_over_ranks(t0.elapsed_time(t1) / 3, world, dev)
    steps = max(20, min(50000, math.ceil(seconds * 1e3 / max(est, 1e-4))))
    barrier(world)
    torch.cuda.synchronize()
    lo = clocks.now()
    t0.record(stream)
    for i in range(steps):
        fn(i % n_sets)
    t1.record(stream)
    torch.cuda.synchronize()
    hi = clocks.now()
    barrier(world)
    return steps, max_over_ranks(t0.elapsed_time(t1), world, dev), clocks.stats(lo, hi)


def run_gemm_sub_results(rank, world, dev, clocks, peaks, seconds):
    from causal_attention_fwd_attn_b200 import _lib

    out = []
    s = torch.cuda.current_stream(dev).cuda_stream
    for name, tokens, din, dout, prod in GEMM_SUB_RESULTS:
        set_bytes = 2 * (tokens * din + dout * din + tokens * dout)
        n_sets = max(2, math.ceil(3 * L2_BYTES / set_bytes))
        sets = []
        for k in range(n_sets):
            seed = 9000 + 10 * k + 97 * rank
            sets.append({"x": wl.gaussian_bf16((tokens, din), 1.0, seed).to(dev),
                         "w": wl.gaussian_bf16((dout, din), 1.0, seed + 1).to(dev),
                         "dy": wl.gaussian_bf16((tokens, dout), 1.0, seed + 2).to(dev)})
        if prod == "fwd":
            y = torch.empty((tokens, dout), dtype=torch.bfloat16, device=dev)

            def fn(i):
                x = sets[i]
                _lib.check(_lib.forge_linear_fwd(x["x"].data_ptr(), x["w"].data_ptr(),
                                                 y.data_ptr(), tokens, din, dout, 0, s), name)
        elif prod == "dx":
            y = torch.empty((tokens, din), dtype=torch.bfloat16, device=dev)

            def fn(i):
                x = sets[i]
                _lib.check(_lib.forge_linear_bwd_dx(x["dy"].data_ptr(), x["w"].data_ptr(),
                                                    y.data_ptr(), tokens, din, dout, 0, s), name)
        else:
            y = torch.empty((dout, din), dtype=torch.float32, device=dev)

            def fn(i):
                x = sets[i]
                _lib.check(_lib.forge_linear_bwd_dw(x["dy"].data_ptr(), x["x"].data_ptr(),
                                                    y.data_ptr(), tokens, din, dout, 0, 0, 0,
                                                    s), name)
        steps, ms, clk = time_loop(fn, n_sets, world, dev, clocks, seconds)
        tf = job_tflops(gemm_flops(tokens, din, dout), steps, world, ms)
        out.append({"workload": name, "kind": "gemm", "tokens": tokens, "in": din, "out": dout,
                    "product": prod, "steps": steps, "ms_per_step": round(ms / steps, 4),
                    "value": round(tf, 2), "unit": UNIT,
                    "frac_of_bf16_peak": round(tf / world / peaks["bf16_tflops"], 4),
                    "split_k": (_lib.forge_linear_split_k(tokens, din, dout)
                                if prod == "dw" else None),
                    "clocks": {k: clk.get(k) for k in ("sm_mhz", "samples", "reasons")}})
        del sets, y
        torch.cuda.empty_cache()
    return out


def run_adamw_sub_result(rank, world, dev, clocks, peaks, seconds):
    """One AdamW step over GPT-2-small-shaped parameters (148 tensors, 124.4M values):
    algorithmic bytes 32 per parameter (norm pass reads the gradient; the update reads
    parameter, gradient and both moments and writes parameter and both moments)."""
    from causal_attention_fwd_attn_b200 import _lib

    shapes = wl.gpt2small_param_shapes()
    host = wl.make_adamw_inputs(shapes, 7000 + rank)
    t = [{k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
         for x in host]
    del host
    n_params = sum(x["param"].numel() for x in t)
    table = [(x["param"].data_ptr(), x["grad"].data_ptr(), x["exp_avg"].data_ptr(),
              x["exp_avg_sq"].data_ptr(), x["param"].numel(), int(x["decay"])) for x in t]
    ws_n = _lib.forge_adamw_workspace_size(len(table))
    ws = torch.empty(ws_n, dtype=torch.uint8, device=dev)
    s = torch.cuda.current_stream(dev).cuda_stream
    state = {"step": 0}

    def fn(i):
        state["step"] += 1
        _lib.check(_lib.forge_adamw_step(table, 3e-4, 0.9, 0.95, 1e-8, 0.1, state["step"], 1.0,
                                         None, ws.data_ptr(), ws_n, s), "adamw")

    steps, ms, clk = time_loop(fn, 1, world, dev, clocks, seconds)
    per_step = ms / steps
    gbs = 32.0 * n_params / (per_step * 1e-3) / 1e9
    res = {"workload": "adamw_gpt2small_124m", "kind": "adamw", "tensors": len(table),
           "params": n_params, "steps": steps, "ms_per_step": round(per_step, 4),
           "value": round(gbs * world, 1), "unit": "GB/s",
           "frac_of_hbm_peak": round(gbs / peaks["hbm_gbs"], 4),
           "algorithmic_bytes_per_step": 32 * n_params,
           "clocks": {k: clk.get(k) for k in ("sm_mhz", "samples", "reasons")}}
    del t, ws
    torch.cuda.empty_cache()
    return res


def run_ours(args, rank, world, local_rank):
    from causal_attention_fwd_attn_b200 import _lib

    ci, w = find_workload(args.workload)
    mode = args.mode or w.mode
    causal = w.causal
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks = measured_peaks()
    clocks = ClockSampler(local_rank).start()
    try:
        sets = input_sets(ci, w, rank, dev)
        p = Pass(w, mode, causal, dev)
        max_ms, avg, clk = timed_run(p, sets, args.warmup, args.steps, world, dev, clocks)
        del sets
        torch.cuda.empty_cache()
        # ---- end to end through the public C ABI with host buffers (pinned) ------
        e2e = None if args.no_e2e else run_e2e(args, w, ci, mode, causal, dev, p, world)
        subs = None
        which = args.sub_results
        if which != "none":
            secs = args.sub_seconds
            subs = []
            if which in ("all", "attention"):
                subs += run_sub_results(rank, world, dev, clocks, peaks, 3, secs)
            if which in ("all", "gemm"):
                subs += run_gemm_sub_results(rank, world, dev, clocks, peaks, secs)
            if which in ("all", "adamw"):
                subs.append(run_adamw_sub_result(rank, world, dev, clocks, peaks, secs))
    finally:
        clocks.stop()
    if rank != 0:
        return None
    traffic = recorded_traffic("attn_bwd_dkdv", f"{w.name}/{mode}")
    return ours_line(w, mode, causal, args.steps, args.warmup, world, max_ms, avg, clk, e2e,
                     p.launches_per_step, peaks, traffic,
                     os.path.relpath(_lib.library_path(), ROOT), subs)


def run_e2e(args, w, ci, mode, causal, dev, p, world):
    """Same metric through the public C ABI (forge_attn_fwd_ex, forge_attn_bwd_ex), with
    each step's inputs copied from pinned host memory and all its outputs (O, LSE, dQ,
    dK, dV) copied back, all inside the timed region.  The copies run on streams of
    their own, as a caller would drive the API: step k+1's inputs go up and step
    k-1's outputs come down while step k computes (two device buffer sets)."""
    L = p.lib
    B, H, T, d = w.B, w.H, w.T, w.d
    x = wl.make_inputs(ci, w, seed_offset=7)
    host_in = {n: t.pin_memory() for n, t in x.items()}
    dev_in = [{n: torch.empty_like(t, device=dev) for n, t in x.items()} for _ in range(2)]
    out0 = {"o": p.o, "lse": p.lse, "dq": p.dq, "dk": p.dk, "dv": p.dv}
    dev_out = [out0, {n: torch.empty_like(t) for n, t in out0.items()}]
    host_out = {n: torch.empty_like(t, device="cpu").pin_memory() for n, t in out0.items()}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    comp = p.stream
    up = torch.cuda.Stream(device=dev)
    down = torch.cuda.Stream(device=dev)
    s = comp.cuda_stream

    def ev():
        return torch.cuda.Event()

    def run(steps, first_event=None):
        """Issues `steps` pipelined steps; returns the event that completes the last
        download (on the compute stream's timeline once waited for)."""
        in_ready, comp_done, out_done = {}, {}, {}
        if first_event is not None:
            up.wait_event(first_event)
            down.wait_event(first_event)
        for k in range(steps):
            b = k % 2
            with torch.cuda.stream(up):
                if k >= 2:
                    up.wait_event(comp_done[k - 2])      # buffer set b's inputs are free
                for n in host_in:
                    dev_in[b][n].copy_(host_in[n], non_blocking=True)
                in_ready[k] = ev()
                in_ready[k].record(up)
            comp.wait_event(in_ready[k])
            if k >= 2:
                comp.wait_event(out_done[k - 2])         # buffer set b's outputs are read
            xin = p.to_fp16(dev_in[b]) if p.fp16 else dev_in[b]
            q, kk, v, dO = (xin[n] for n in ("q", "k", "v", "dO"))
            o = dev_out[b]
            L.check(L.forge_attn_fwd_ex(q.data_ptr(), kk.data_ptr(), v.data_ptr(),
                                        o["o"].data_ptr(), o["lse"].data_ptr(), B, H, T, d,
                                        w.scale, causal, p.fwd_flags, s), "fwd")
            L.check(L.forge_attn_bwd_ex(q.data_ptr(), kk.data_ptr(), v.data_ptr(),
                                        o["o"].data_ptr(), dO.data_ptr(), o["lse"].data_ptr(),
                                        o["dq"].data_ptr(), o["dk"].data_ptr(),
                                        o["dv"].data_ptr(), p.ws.data_ptr(), p.ws_n, B, H, T, d,
                                        w.scale, causal, p.bwd_flags, s), "bwd")
            comp_done[k] = ev()
            comp_done[k].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(comp_done[k])
                for n in host_out:
                    host_out[n].copy_(o[n], non_blocking=True)
                out_done[k] = ev()
                out_done[k].record(down)
        comp.wait_event(out_done[steps - 1])
        comp.wait_event(in_ready[steps - 1])

    steps = max(3, min(args.steps, 20))
    run(2)
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(comp)
    run(steps, first_event=t0)
    t1.record(comp)
    torch.cuda.synchronize()
    p.check_device("in the end-to-end run")
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    fwd_flops, bwd_flops = causal_flops(w, causal)
    value = job_tflops(fwd_flops + bwd_flops, steps, world, ms)
    return {"value": round(value, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": round(ms / steps, 4),
            "api": "forge_attn_fwd_ex + forge_attn_bwd_ex",
            "copies": "own streams: step k+1's inputs up and step k-1's outputs down while "
                      "step k computes (two device buffer sets)"}


# ---------------------------------------------------------- CPU oracle leg ----
class OracleSampler:
    """Times the fp64 oracle (forward + backward, the full T x T definition) on whole
    heads of a workload, on the host's cores, cycling through the workload's heads.
    The oracle is single-threaded per head; a task is a run of consecutive head passes
    on one thread, and tasks run concurrently, one per thread."""

    def __init__(self, w, ci, threads, causal=None):
        import oracle

        self.w = w
        self.causal = w.causal if causal is None else causal
        self.orc = oracle.default()
        x = wl.make_inputs(ci)
        self.f = {n: x[n].double().numpy() for n in x}
        self.heads = [(b, h) for b in range(w.B) for h in range(w.H)]
        self.threads = max(1, threads)
        self.cursor = 0
        self.head_s = None  # seconds per head pass on one thread, once measured

    def _take(self, n):
        hs = [self.heads[(self.cursor + j) % len(self.heads)] for j in range(n)]
        self.cursor = (self.cursor + n) % len(self.heads)
        return hs

    def _one(self, bh):
        f, w, orc = self.f, self.w, self.orc
        b, h = bh
        orc.fwd_head(f["q"][b, h], f["k"][b, h], f["v"][b, h], w.scale, self.causal)
        orc.bwd_head(f["q"][b, h], f["k"][b, h], f["v"][b, h], f["dO"][b, h], w.scale,
                     self.causal)

    def run_tasks(self, n_tasks, heads_per_task):
        """Runs n_tasks tasks of heads_per_task head passes each, concurrently on
        min(threads, n_tasks) threads; returns (wall seconds, threads used)."""
        from concurrent.futures import ThreadPoolExecutor

        tasks = [self._take(heads_per_task) for _ in range(n_tasks)]
        threads = min(self.threads, n_tasks)
        t = time.perf_counter()
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(lambda hs: [self._one(bh) for bh in hs], tasks))
        wall = time.perf_counter() - t
        if heads_per_task == 1 and n_tasks <= threads:
            self.head_s = wall
        return wall, threads

    def flops_per_head(self):
        fwd, bwd = causal_flops(self.w, self.causal)
        return (fwd + bwd) / self.w.BH

    def sample(self, budget_s):
        """(TFLOP/s in the workload's FLOP convention, threads used, description, wall
        seconds) of one sample of about budget_s seconds with every thread busy: a first
        round of one head pass per thread measures the rate; if that round already took
        most of the budget it is the sample, else a second round of longer tasks is."""
        n = min(self.threads, len(self.heads))
        wall, threads = self.run_tasks(n, 1)
        per_task = 1
        if wall < 0.5 * budget_s:
            per_task = max(1, int(budget_s / max(self.head_s, 1e-6)))
            wall, threads = self.run_tasks(n, per_task)
        passes = n * per_task
        value = self.flops_per_head() * passes / wall / 1e12
        desc = (f"{passes} head passes over the {self.w.BH} heads of {self.w.name} "
                f"(T={self.w.T}, d={self.w.d}), fp64 oracle forward + backward, "
                f"{wall:.2f} s on {threads} threads")
        return value, threads, desc, wall


def run_reference(args, rank, world):
    """The oracle as it stands, timed on the host cores.  A step is a bounded sample of
    the workload: a run of consecutive whole-head passes (forward + backward) on one
    thread.  The warm-up steps are one head pass each and also measure the per-head
    time; the timed steps are sized so that the timed phase takes about
    args.reference_seconds, and run concurrently, one per thread."""
    if rank != 0:
        return None
    ci, w = find_workload(args.workload)
    mode = getattr(args, "mode", None) or w.mode
    threads = max(1, os.cpu_count() or 1)
    sampler = OracleSampler(w, ci, threads)
    t_warm, _ = sampler.run_tasks(args.warmup, 1)
    head_s = sampler.head_s or t_warm
    rounds = math.ceil(args.steps / min(threads, args.steps))
    per_step = max(1, int(args.reference_seconds / (rounds * head_s)))
    wall, used = sampler.run_tasks(args.steps, per_step)
    passes = args.steps * per_step
    value = sampler.flops_per_head() * passes / wall / 1e12
    desc = (f"{args.steps} steps of {per_step} head passes each over the {w.BH} heads of "
            f"{w.name} (T={w.T}, d={w.d}), fp64 oracle forward + backward, run "
            f"concurrently: {wall:.2f} s on {used} threads")
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(wall * 1e3 / args.steps, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": config_of(w, mode, w.causal, world),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": used,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 300; 20 for --impl reference)")
    ap.add_argument("--warmup", type=int, default=None,
                    help="untimed warm-up steps, at least 3 (default 10; 5 for --impl reference)")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--mode", choices=sorted(wl.MODES), default=None,
                    help="default: the mode the workload's parity tests use")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-baseline-seconds", type=float, default=12.0,
                    help="budget of the oracle sample timed beside the GPU run (rank 0, N=1)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sub-results", choices=["all", "attention", "gemm", "adamw", "none"],
                    default="all", help="which sub-results to time beside the headline")
    ap.add_argument("--no-sub-results", action="store_true", help="same as --sub-results none")
    ap.add_argument("--sub-seconds", type=float, default=SUB_RESULT_SECONDS,
                    help="GPU time of each sub-result's timed loop (20 steps at least)")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end (host buffers) measurement")
    ap.add_argument("--reference-seconds", type=float, default=90.0,
                    help="--impl reference: about how long the timed steps take in all "
                         "(each step is at least one head pass)")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = 20 if args.impl == "reference" else 300
    if args.warmup is None:
        args.warmup = 5 if args.impl == "reference" else 10
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.steps < 1:
        raise SystemExit("--steps must be at least 1")
    if args.no_sub_results:
        args.sub_results = "none"

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
            v, cores, desc, _ = OracleSampler(w, ci, os.cpu_count() or 1).sample(
                args.cpu_baseline_seconds)
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
