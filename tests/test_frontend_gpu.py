"""The torch front end on the GPU: the fp16-operand route (bf16 tensors converted with
to_fp16, fp32 outputs) against the fp64 oracle, output dtypes, and to_fp16's range
check."""
import pytest
import torch

import oracle
from causal_attention_fwd_attn_b200 import attention as A
from causal_attention_fwd_attn_b200 import workloads as wl
from tests.gpu_helpers import as_f64, assert_close

pytestmark = pytest.mark.gpu


def test_fp16_route_through_the_front_end():
    w = wl.custom(2, 3, 300, 128)
    x = wl.make_inputs(0, w, seed_offset=83)
    dev = torch.device("cuda", 0)
    q, k, v, dO = (A.to_fp16(x[n].to(dev)) for n in ("q", "k", "v", "dO"))
    o, lse = A.attn_fwd(q, k, v, o_dtype=torch.float32)
    dq, dk, dv = A.attn_bwd(q, k, v, o, dO, lse, grad_dtype=torch.float32)
    A.check_device_error()
    f = as_f64(x)
    orc = oracle.default()
    ro, rlse = orc.fwd(f["q"], f["k"], f["v"], w.scale, w.causal, threads=4)
    rdq, rdk, rdv = orc.bwd(f["q"], f["k"], f["v"], f["dO"], w.scale, w.causal, threads=4)
    for n, got, ref in (("o", o, ro), ("lse", lse, rlse), ("dq", dq, rdq), ("dk", dk, rdk),
                        ("dv", dv, rdv)):
        assert_close(n, got.cpu().numpy(), ref, "front end, fp16 operands")


def test_default_output_dtypes_follow_the_inputs():
    dev = torch.device("cuda", 0)
    g = torch.Generator().manual_seed(3)
    for dt in (torch.bfloat16, torch.float16):
        q = torch.randn((1, 2, 130, 64), generator=g).to(dt).to(dev)
        o, lse = A.attn_fwd(q, q, q)
        dq, dk, dv = A.attn_bwd(q, q, q, o, q, lse)
        assert o.dtype == dq.dtype == dk.dtype == dv.dtype == dt
        assert lse.dtype == torch.float32
    A.check_device_error()


def test_to_fp16_refuses_values_beyond_fp16s_range():
    dev = torch.device("cuda", 0)
    x = torch.ones(64, dtype=torch.bfloat16, device=dev)
    x[5] = 70000.0
    with pytest.raises(ValueError, match="beyond fp16"):
        A.to_fp16(x)
    assert torch.equal(A.to_fp16(torch.ones(9, dtype=torch.bfloat16, device=dev)).cpu(),
                       torch.ones(9, dtype=torch.float16))
