"""Shared helpers of the GPU tests: run the CUDA path through the C ABI and
compare with the oracle under the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

from causal_attention_fwd_attn_b200 import _lib
from causal_attention_fwd_attn_b200 import workloads as wl

# Tolerances: relative L2 <= 1e-2 and max abs <= 2e-2 on O, dQ, dK, dV; both <= 1e-3
# on LSE.
TOL = {"o": (1e-2, 2e-2), "dq": (1e-2, 2e-2), "dk": (1e-2, 2e-2), "dv": (1e-2, 2e-2),
       "lse": (1e-3, 1e-3)}


def errors(gpu, ref):
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(r)
    rel = np.linalg.norm(g - r) / den if den > 0 else np.linalg.norm(g - r)
    return float(rel), float(np.max(np.abs(g - r))) if g.size else 0.0


def assert_close(name, gpu, ref, what=""):
    rel, mx = errors(gpu, ref)
    trel, tabs = TOL[name]
    assert np.all(np.isfinite(np.asarray(gpu, dtype=np.float64))), f"{what} {name}: non-finite"
    assert rel <= trel and mx <= tabs, \
        f"{what} {name}: rel-L2 {rel:.3e} (tol {trel}), max-abs {mx:.3e} (tol {tabs})"
    return rel, mx


def to_fp16_on_device(t, s):
    """bf16 device tensor -> fp16 through the library's conversion (no value may leave
    fp16's range)."""
    out = torch.empty_like(t, dtype=torch.float16)
    over = torch.zeros(1, dtype=torch.int32, device=t.device)
    _lib.check(_lib.forge_attn_bf16_to_fp16(t.data_ptr(), out.data_ptr(), t.numel(),
                                            over.data_ptr(), s), "bf16_to_fp16")
    assert int(over.item()) == 0, "values beyond fp16's range"
    return out


def run_gpu(x, scale, causal, o_dtype=None, grad_dtype=None, bwd=True, precise=False,
            fp16=False):
    """Forward (and backward) through the C ABI on cuda:0.  x: dict of CPU bf16 (or fp16:
    the fp16-operand mode) tensors; fp16=True converts bf16 inputs to fp16 on the device
    with the library first.  Outputs default to the kernels' input dtype.  With an fp32 O
    the backward reads that fp32 O for its D pre-pass."""
    dev = torch.device("cuda", 0)
    s = torch.cuda.current_stream(dev).cuda_stream
    q, k, v, dO = (x[n].to(dev) for n in ("q", "k", "v", "dO"))
    if fp16:
        q, k, v, dO = (to_fp16_on_device(t, s) for t in (q, k, v, dO))
    B, H, T, d = q.shape
    o_dtype = o_dtype or q.dtype
    grad_dtype = grad_dtype or q.dtype
    pflag = (_lib.PRECISE if precise else 0) | (_lib.FP16 if q.dtype == torch.float16 else 0)
    o = torch.empty((B, H, T, d), dtype=o_dtype, device=dev)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    fflags = (_lib.OUT_F32 if o_dtype == torch.float32 else 0) | pflag
    _lib.check(_lib.forge_attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                      lse.data_ptr(), B, H, T, d, scale, causal, fflags, s),
               "fwd")
    out = {"o": o, "lse": lse}
    if bwd:
        ws_n = _lib.forge_attn_bwd_workspace_size(B, H, T, d)
        ws = torch.empty(ws_n, dtype=torch.uint8, device=dev)
        dq, dk, dv = (torch.empty((B, H, T, d), dtype=grad_dtype, device=dev) for _ in range(3))
        bflags = ((_lib.OUT_F32 if grad_dtype == torch.float32 else 0)
                  | (_lib.O_IN_F32 if o_dtype == torch.float32 else 0) | pflag)
        _lib.check(_lib.forge_attn_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                          o.data_ptr(), dO.data_ptr(), lse.data_ptr(),
                                          dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                          ws.data_ptr(), ws_n, B, H, T, d, scale, causal,
                                          bflags, s), "bwd")
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    st, detail = _lib.forge_attn_check_device_error(s)
    assert st == _lib.OK, f"device wait timed out: 0x{detail:08x}"
    return {n: t.float().cpu().numpy() for n, t in out.items()}


def mode_kwargs(mode):
    """run_gpu keyword arguments of a workload mode ("default" or "accuracy")."""
    m = wl.MODES[mode]
    return dict(o_dtype=torch.float32 if m["o_f32"] else torch.bfloat16,
                grad_dtype=torch.float32 if m["grad_f32"] else torch.bfloat16,
                precise=m["precise"], fp16=m["fp16"])


def oracle_threads(T):
    """Host threads for the full oracle at sequence length T: one head per thread,
    capped by the memory its T x T buffers take (three fp64 matrices per head)."""
    import os

    import psutil

    per_head = 3 * 8 * T * T + (64 << 20)
    avail = psutil.virtual_memory().available
    return max(1, min(os.cpu_count() or 1, int(0.7 * avail // per_head)))


def as_f64(x):
    return {n: t.double().numpy() for n, t in x.items()}
