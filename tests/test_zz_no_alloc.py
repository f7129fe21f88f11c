"""forge_attn_bwd_noalloc: the backward for callers that cannot allocate device
memory -- a process whose memory budget is fixed once it starts, a plugin that is
handed raw device pointers but no allocator, a latency-critical loop that must stay
off the allocator.  Its scratch is a fixed array inside the library, so it must give
the gradients of forge_attn_bwd with a caller-allocated workspace, call after call.

This file is collected last on purpose: a run that stops at its first failure has
already run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
from causal_attention_fwd_attn_b200 import _lib, build
from causal_attention_fwd_attn_b200 import workloads as wl
from tests.gpu_helpers import TOL, as_f64, assert_close, errors

P = 4096  # a 16-byte aligned fake address; never dereferenced (rejected first)


def test_noalloc_refuses_sizes_beyond_its_array():
    build.build()
    # B=2 H=16 T=4096 d=128 needs about 68 MB of scratch, more than the 64 MiB array
    assert _lib.forge_attn_bwd_workspace_size(2, 16, 4096, 128) > _lib.NOALLOC_SCRATCH_BYTES
    args = [P] * 9 + [2, 16, 4096, 128, 0.1, 1, None]
    assert _lib.forge_attn_bwd_noalloc(*args) == _lib.ERR_WORKSPACE
    # ordinary argument errors keep their codes
    assert _lib.forge_attn_bwd_noalloc(*([0] + [P] * 8 + [1, 1, 8, 64, 0.1, 1, None])) == \
        _lib.ERR_INVALID_ARG
    assert _lib.forge_attn_bwd_noalloc(*([P] * 9 + [1, 1, 8, 96, 0.1, 1, None])) == \
        _lib.ERR_UNSUPPORTED
    assert _lib.forge_attn_bwd_noalloc(*([P + 8] + [P] * 8 + [1, 1, 8, 64, 0.1, 1, None])) == \
        _lib.ERR_MISALIGNED


def _backward_both_ways(x, w, dev, s):
    q, k, v, dO = (x[n].to(dev) for n in ("q", "k", "v", "dO"))
    B, H, T, d = q.shape
    o = torch.empty_like(q)
    lse = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    _lib.check(_lib.forge_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   lse.data_ptr(), B, H, T, d, w.scale, 1, s), "fwd")
    ref = [torch.empty_like(q) for _ in range(3)]
    ws_n = _lib.forge_attn_bwd_workspace_size(B, H, T, d)
    ws = torch.empty(ws_n, dtype=torch.uint8, device=dev)
    _lib.check(_lib.forge_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   dO.data_ptr(), lse.data_ptr(), ref[0].data_ptr(),
                                   ref[1].data_ptr(), ref[2].data_ptr(), ws.data_ptr(), ws_n, B,
                                   H, T, d, w.scale, 1, s), "bwd")
    got = [torch.full_like(q, float("nan")) for _ in range(3)]
    _lib.check(_lib.forge_attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                           dO.data_ptr(), lse.data_ptr(), got[0].data_ptr(),
                                           got[1].data_ptr(), got[2].data_ptr(), B, H, T, d,
                                           w.scale, 1, s), "bwd_noalloc")
    torch.cuda.synchronize()
    st, detail = _lib.forge_attn_check_device_error(s)
    assert st == _lib.OK, hex(detail)
    return ([t.float().cpu().numpy() for t in ref], [t.float().cpu().numpy() for t in got])


# (1, 96, 384, 64): 288 key-tile items, about two per persistent CTA
@pytest.mark.gpu
@pytest.mark.parametrize("shape", [(2, 3, 300, 64), (1, 4, 513, 128), (1, 96, 384, 64)])
def test_noalloc_matches_workspace_backward_twice(shape):
    dev = torch.device("cuda", 0)
    s = torch.cuda.current_stream(dev).cuda_stream
    w = wl.custom(*shape)
    orc = oracle.default()
    # two calls in a row on different inputs: the second must not see the first's scratch
    for call in range(2):
        x = wl.make_inputs(0, w, seed_offset=1000 + 37 * call + shape[3])
        ref, got = _backward_both_ways(x, w, dev, s)
        for name, a, b in zip(("dq", "dk", "dv"), got, ref):
            assert np.all(np.isfinite(a)), f"call {call} {name}"
            rel, mx = errors(a, b)
            trel, tabs = TOL[name]
            assert rel <= trel and mx <= tabs, f"call {call} {name}: {rel:.3e} {mx:.3e}"
        # dK and dV come from the same deterministic kernel with the same inputs
        assert np.array_equal(got[1], ref[1]) and np.array_equal(got[2], ref[2])
        # and all three against the fp64 oracle on the same inputs
        f = as_f64(x)
        exact = orc.bwd(f["q"], f["k"], f["v"], f["dO"], w.scale, 1, threads=8)
        for name, a, b in zip(("dq", "dk", "dv"), got, exact):
            assert_close(name, a, b, f"noalloc call {call} {w.describe()}")
