"""Bounded device-side waits: a wait that nothing completes gives up, reports
FORGE_ATTN_ERR_TIMEOUT through forge_attn_check_device_error, and leaves the
context usable (GPU).  No fault, trap or hang is involved: the kernel returns on
its own after the wait limit."""
import numpy as np
import pytest
import torch

from causal_attention_fwd_attn_b200 import _lib
from causal_attention_fwd_attn_b200 import workloads as wl
from tests.gpu_helpers import run_gpu

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_is_reported_and_cleared():
    s = torch.cuda.current_stream().cuda_stream
    st, _ = _lib.forge_attn_check_device_error(s)
    assert st == _lib.OK
    _lib.check(_lib.forge_probe_wait_timeout(2_000_000, s), "probe")  # 2 ms limit
    st, detail = _lib.forge_attn_check_device_error(s)
    assert st == _lib.ERR_TIMEOUT
    assert detail & 0x80000000
    assert (detail >> 20) & 0x7FF == 0x7FF  # the probe's wait site
    st, detail = _lib.forge_attn_check_device_error(s)
    assert st == _lib.OK and detail == 0


def test_context_usable_after_a_timeout():
    s = torch.cuda.current_stream().cuda_stream
    _lib.check(_lib.forge_probe_wait_timeout(1_000_000, s), "probe")
    assert _lib.forge_attn_check_device_error(s)[0] == _lib.ERR_TIMEOUT
    w = wl.custom(1, 1, 64, 64)
    got = run_gpu(wl.make_inputs(0, w, seed_offset=99), w.scale, 1)
    assert np.all(np.isfinite(got["o"]))


def test_host_errors_do_not_launch():
    s = torch.cuda.current_stream().cuda_stream
    assert _lib.forge_attn_fwd(0, 0, 0, 0, 0, 1, 1, 8, 64, 0.1, 1, s) == _lib.ERR_INVALID_ARG
    assert _lib.forge_attn_check_device_error(s)[0] == _lib.OK
