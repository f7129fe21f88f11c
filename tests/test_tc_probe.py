"""One tensor-core tile in each operand form the attention kernels use, against a
plain torch fp32 product of the same bf16 values (GPU)."""
import pytest
import torch

from causal_attention_fwd_attn_b200 import _lib

pytestmark = pytest.mark.gpu


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("mode", [0, 1, 2, 3])
@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("K", [64, 128])
def test_probe_tile(mode, N, K):
    dev = torch.device("cuda", 0)
    if mode == 3:
        a = _rand((K, 128), 1 + N + K)
        ref_a = a.float().T
    else:
        a = _rand((128, K), 1 + N + K)
        ref_a = a.float()
    if mode == 0:
        b = _rand((N, K), 2 + N + K)
        ref = ref_a @ b.float().T
    else:
        b = _rand((K, N), 2 + N + K)
        ref = ref_a @ b.float()
    ga, gb = a.to(dev), b.to(dev)
    out = torch.full((128, N), float("nan"), device=dev)
    s = torch.cuda.current_stream().cuda_stream
    _lib.check(_lib.forge_probe_mma(ga.data_ptr(), gb.data_ptr(), out.data_ptr(), N, K, mode, s),
               "probe")
    torch.cuda.synchronize()
    st, detail = _lib.forge_attn_check_device_error(s)
    assert st == _lib.OK, hex(detail)
    got = out.cpu()
    assert torch.allclose(got, ref, rtol=1e-4, atol=1e-3), \
        f"mode {mode} N {N} K {K}: max err {(got - ref).abs().max().item()}"
