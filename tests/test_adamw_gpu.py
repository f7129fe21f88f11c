"""The fused multi-tensor AdamW step (CUDA, through the C ABI) against the fp64 oracle
on the same fp32 inputs (GPU).

Tolerance: the step is a handful of fp32 operations per element, each rounded once
(2^-24 relative), and the clip factor comes from an fp32 norm whose relative error is
about 1e-6.  A result can cancel far below its terms (m = beta1 m + (1 - beta1) g
near zero), so the bound is relative to the element with an absolute floor relative
to the tensor: per element |gpu - ref| <= 1e-5 |ref| + 1e-6 max|ref| (a few fp32
ulps of the tensor's largest terms); the global norm to 1e-5 relative.
"""
import numpy as np
import pytest
import torch

from causal_attention_fwd_attn_b200 import _lib
from causal_attention_fwd_attn_b200 import workloads as wl
from oracle import adamw as oa

pytestmark = pytest.mark.gpu

HP = dict(lr=3e-3, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1)


def run_steps(shapes, seed, steps, max_norms):
    dev = torch.device("cuda", 0)
    s = torch.cuda.current_stream(dev).cuda_stream
    host = wl.make_adamw_inputs(shapes, seed)
    gpu = [{k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in t.items()}
           for t in host]
    ref_p = [t["param"].double().numpy() for t in host]
    ref_m = [t["exp_avg"].double().numpy() for t in host]
    ref_v = [t["exp_avg_sq"].double().numpy() for t in host]
    decay = [t["decay"] for t in host]
    ws_n = _lib.forge_adamw_workspace_size(len(shapes))
    ws = torch.empty(ws_n, dtype=torch.uint8, device=dev)
    norm = torch.empty(1, dtype=torch.float32, device=dev)
    g = torch.Generator().manual_seed(seed + 1)
    for step in range(1, steps + 1):
        if step > 1:  # a fresh gradient every step
            for t in gpu:
                t["grad"] = (torch.randn(t["grad"].shape, generator=g) * 0.01).to(dev)
        grads = [t["grad"].double().cpu().numpy() for t in gpu]
        table = [(t["param"].data_ptr(), t["grad"].data_ptr(), t["exp_avg"].data_ptr(),
                  t["exp_avg_sq"].data_ptr(), t["param"].numel(), int(t["decay"])) for t in gpu]
        _lib.check(_lib.forge_adamw_step(table, step=step, max_norm=max_norms[step - 1],
                                         grad_norm_out=norm.data_ptr(), workspace=ws.data_ptr(),
                                         workspace_bytes=ws_n, stream=s, **HP), "adamw")
        ref_p, ref_m, ref_v, ref_norm = oa.adamw_step(ref_p, grads, ref_m, ref_v, decay,
                                                       step=step, max_norm=max_norms[step - 1],
                                                       **HP)
        torch.cuda.synchronize()
        assert norm.item() == pytest.approx(ref_norm, rel=1e-5), f"step {step} norm"
        for i, t in enumerate(gpu):
            for name, ref in (("param", ref_p[i]), ("exp_avg", ref_m[i]),
                              ("exp_avg_sq", ref_v[i])):
                got = t[name].double().cpu().numpy()
                np.testing.assert_allclose(got, ref, rtol=1e-5,
                                           atol=1e-6 * float(np.max(np.abs(ref))),
                                           err_msg=f"step {step} tensor {i} {name}")
    return ref_norm


def test_ragged_tensors_three_steps_with_and_without_clipping():
    shapes = [(1,), (3,), (5, 7), (1000,), (65536 + 7,), (300, 701), (2, 3, 4)]
    # step 1 unclipped, step 2 clipped hard, step 3 with clipping disabled
    run_steps(shapes, 11, 3, [1e9, 0.05, 0.0])


def test_more_tensors_than_one_launch_holds():
    n = _lib.ADAMW_MAX_TENSORS_PER_LAUNCH + 45
    shapes = [((i * 37) % 500 + 1,) if i % 3 else (i % 7 + 1, 19) for i in range(n)]
    run_steps(shapes, 12, 2, [0.1, 1e9])


def test_gpt2_small_parameter_set():
    run_steps(wl.gpt2small_param_shapes(), 13, 1, [1.0])
