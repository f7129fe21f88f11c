"""The torch front end's argument checks, on the CPU: the C ABI sees raw pointers,
so a caller-supplied buffer of the wrong device, dtype, shape or layout must be
refused in Python before any pointer is passed on."""
import pytest
import torch

from causal_attention_fwd_attn_b200 import attention as A

CPU = torch.device("cpu")


def test_a_matching_tensor_passes():
    t = torch.empty((2, 3, 5, 64), dtype=torch.bfloat16)
    assert A._check_tensor(t, "t", (2, 3, 5, 64), (torch.bfloat16,), CPU) is t


@pytest.mark.parametrize("make,msg", [
    (lambda: torch.empty((2, 3, 5, 64), dtype=torch.float16), "dtype"),
    (lambda: torch.empty((2, 3, 5, 128), dtype=torch.bfloat16), "shape"),
    (lambda: torch.empty((2, 3, 64, 5), dtype=torch.bfloat16).transpose(2, 3), "contiguous"),
    (lambda: torch.empty((2, 3, 5, 64), dtype=torch.bfloat16, device="meta"), "meta"),
    (lambda: [0.0] * 4, "torch.Tensor"),
])
def test_a_wrong_tensor_is_refused(make, msg):
    with pytest.raises(ValueError, match=msg):
        A._check_tensor(make(), "t", (2, 3, 5, 64), (torch.bfloat16,), CPU)


def test_fp32_outputs_are_accepted_where_allowed():
    t = torch.empty((1, 1, 4, 64), dtype=torch.float32)
    assert A._check_tensor(t, "out", (1, 1, 4, 64), A._GRAD_DTYPES, CPU) is t


def test_cpu_inputs_are_refused_before_any_library_call():
    q = torch.zeros((1, 1, 8, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        A.attn_fwd(q, q, q)
    with pytest.raises(ValueError, match="CUDA"):
        A.attn_bwd(q, q, q, q, q, torch.zeros((1, 1, 8)))
    with pytest.raises(ValueError, match=r"\[B, H, T, d\]"):
        A.attn_fwd(torch.zeros((8, 64), dtype=torch.bfloat16), q, q)


def test_k_v_must_share_q_dtype():
    # what _check_qkv applies to k and v (it needs CUDA tensors itself)
    q = torch.zeros((1, 1, 8, 64), dtype=torch.bfloat16)
    k = torch.zeros((1, 1, 8, 64), dtype=torch.float16)
    with pytest.raises(ValueError, match="dtype"):
        A._check_tensor(k, "k", q.shape, (q.dtype,), CPU)


def test_fp16_inputs_take_fp16_or_fp32_outputs():
    assert A._out_dtypes(torch.float16) == (torch.float16, torch.float32)
    assert A._out_dtypes(torch.bfloat16) == (torch.bfloat16, torch.float32)


def test_to_fp16_refuses_cpu_tensors():
    with pytest.raises(ValueError, match="CUDA"):
        A.to_fp16(torch.zeros(8, dtype=torch.bfloat16))
