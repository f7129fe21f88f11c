"""The bf16 -> fp16 conversion (forge_attn_bf16_to_fp16, through the C ABI) against
IEEE round-to-nearest-even as torch's CPU conversion computes it (GPU).

bf16 has 65536 bit patterns; all of them are converted and compared bit for bit (NaN
only as NaN), together with the count of values beyond fp16's largest finite value
65504, and lengths that leave a tail after the last group of eight values.
"""
import numpy as np
import pytest
import torch

from causal_attention_fwd_attn_b200 import _lib

pytestmark = pytest.mark.gpu


def convert(src_cpu):
    dev = torch.device("cuda", 0)
    s = torch.cuda.current_stream(dev).cuda_stream
    src = src_cpu.to(dev)
    dst = torch.full(src.shape, float("nan"), dtype=torch.float16, device=dev)
    over = torch.zeros(1, dtype=torch.int32, device=dev)
    _lib.check(_lib.forge_attn_bf16_to_fp16(src.data_ptr(), dst.data_ptr(), src.numel(),
                                            over.data_ptr(), s), "bf16_to_fp16")
    torch.cuda.synchronize()
    return dst.cpu(), int(over.item())


def check_against_ieee(src):
    got, over = convert(src)
    want = src.to(torch.float16)
    g = got.view(torch.int16).numpy()
    w = want.view(torch.int16).numpy()
    nan = np.isnan(src.float().numpy())
    assert np.array_equal(np.isnan(got.float().numpy()), nan)
    assert np.array_equal(g[~nan], w[~nan])
    beyond = np.abs(src.float().numpy()) > 65504.0
    assert over == int(np.count_nonzero(beyond & ~nan))


def test_every_bf16_bit_pattern():
    bits = torch.arange(-32768, 32768, dtype=torch.int32).to(torch.int16)
    check_against_ieee(bits.view(torch.bfloat16))


@pytest.mark.parametrize("n", [1, 7, 8, 9, 15, 4101, 65533])
def test_lengths_with_a_tail(n):
    g = torch.Generator().manual_seed(n)
    x = (torch.randn(n, generator=g) * 3000).to(torch.bfloat16)
    x[:: 97] = torch.tensor(70000.0).to(torch.bfloat16)  # some beyond fp16's range
    check_against_ieee(x)


def test_values_inside_the_normal_range_convert_exactly():
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(1 << 16, generator=g) * 50).to(torch.bfloat16)
    x = x[(x.float().abs() >= 2.0 ** -14) | (x == 0)]
    got, over = convert(x)
    assert over == 0
    assert torch.equal(got.to(torch.bfloat16), x)
