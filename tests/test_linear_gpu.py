"""The projection GEMMs (tcgen05, through the C ABI) against the fp64 oracle on the same
seeded bf16 (or fp16) inputs (GPU), over whole outputs.

Tolerances, from the arithmetic: the products accumulate in fp32, whose error is far
below 1e-5 of the outputs' rms at these depths; a 16-bit output adds one
round-to-nearest of at most 2^-9 relative.  So per element
  16-bit outputs:  |gpu - ref| <= 2^-8 |ref| + 1e-3 rms(ref)
  fp32 outputs:    |gpu - ref| <= 2e-4 rms(ref) + 1e-5 |ref|
and the relative L2 error over the whole output stays below 3e-3 (16-bit) or 2e-5
(fp32).
"""
import numpy as np
import pytest
import torch

from causal_attention_fwd_attn_b200 import _lib
from causal_attention_fwd_attn_b200 import workloads as wl
from oracle import linear as ol

pytestmark = pytest.mark.gpu


def gen(shape, seed, dtype=torch.bfloat16):
    return wl.gaussian_bf16(shape, 1.0, seed, dtype)


def close(got, ref, f32, what):
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(r * r)))
    err = np.abs(g - r)
    rel = float(np.linalg.norm(g - r) / np.linalg.norm(r))
    if f32:
        bound = 2e-4 * rms + 1e-5 * np.abs(r)
        rel_tol = 2e-5
    else:
        bound = 2.0 ** -8 * np.abs(r) + 1e-3 * rms
        rel_tol = 3e-3
    worst = float(np.max(err - bound))
    print(f"{what}: rel-L2 {rel:.2e} max-abs {float(np.max(err)):.3e} rms(ref) {rms:.3f}")
    assert np.all(np.isfinite(g)), what
    assert worst <= 0 and rel <= rel_tol, f"{what}: rel-L2 {rel:.3e}, worst excess {worst:.3e}"


def run(tokens, din, dout, seed, dtype=torch.bfloat16, out_f32=False, split_k=0,
        accumulate=False):
    dev = torch.device("cuda", 0)
    s = torch.cuda.current_stream(dev).cuda_stream
    x, w, dy = gen((tokens, din), seed, dtype), gen((dout, din), seed + 1, dtype), \
        gen((tokens, dout), seed + 2, dtype)
    X, W, DY = (t.to(dev) for t in (x, w, dy))
    odt = torch.float32 if out_f32 else dtype
    flags = (_lib.OUT_F32 if out_f32 else 0) | (_lib.FP16 if dtype == torch.float16 else 0)
    y = torch.empty((tokens, dout), dtype=odt, device=dev)
    dx = torch.empty((tokens, din), dtype=odt, device=dev)
    prior = gen((dout, din), seed + 3, torch.float32).to(dev) if accumulate else None
    dw = prior.clone() if accumulate else torch.full((dout, din), float("nan"), device=dev)
    _lib.check(_lib.forge_linear_fwd(X.data_ptr(), W.data_ptr(), y.data_ptr(), tokens, din, dout,
                                     flags, s), "fwd")
    _lib.check(_lib.forge_linear_bwd_dx(DY.data_ptr(), W.data_ptr(), dx.data_ptr(), tokens, din,
                                        dout, flags, s), "dx")
    _lib.check(_lib.forge_linear_bwd_dw(DY.data_ptr(), X.data_ptr(), dw.data_ptr(), tokens, din,
                                        dout, split_k, int(accumulate),
                                        flags & _lib.FP16, s), "dw")
    torch.cuda.synchronize()
    st, detail = _lib.forge_attn_check_device_error(s)
    assert st == _lib.OK, hex(detail)
    xd, wd, dyd = (t.double().numpy() for t in (x, w, dy))
    what = f"tokens={tokens} in={din} out={dout} {dtype} split_k={split_k}"
    close(y.double().cpu().numpy(), ol.linear_fwd(xd, wd), out_f32, f"Y {what}")
    close(dx.double().cpu().numpy(), ol.linear_bwd_dx(dyd, wd), out_f32, f"dX {what}")
    ref_dw = ol.linear_bwd_dw(dyd, xd)
    if accumulate:
        ref_dw = ref_dw + prior.double().cpu().numpy()
    close(dw.double().cpu().numpy(), ref_dw, True, f"dW {what}")


@pytest.mark.parametrize("shape", [(8, 8, 8), (200, 72, 136), (136, 520, 264), (1000, 64, 520)])
def test_ragged_shapes(shape):
    run(*shape, seed=sum(shape))


def test_gpt2_small_mlp_shapes():
    # B = 8, T = 1024 tokens; the first MLP layer (768 -> 3072) and the second (3072 -> 768)
    run(8192, 768, 3072, seed=31)
    run(8192, 3072, 768, seed=37)


@pytest.mark.parametrize("split_k", [1, 3, 0])
def test_dw_split_k(split_k):
    run(4096, 256, 384, seed=41 + split_k, split_k=split_k)


def test_dw_accumulates_into_existing_gradient():
    run(2048, 192, 320, seed=43, split_k=4, accumulate=True)
    run(2048, 192, 320, seed=47, split_k=1, accumulate=True)


def test_fp32_outputs():
    run(520, 200, 328, seed=53, out_f32=True)


def test_fp16_operands():
    run(1032, 264, 392, seed=59, dtype=torch.float16)


# Shapes whose products take the wider tiles on a 148-SM B200 (by the library's plan
# cost model), with rows and columns that end inside a tile:
#   (3000, 776, 776)    Y and dX on 128 x 256 tiles (dW 128 x 128, split 3)
#   (3000, 2056, 1544)  Y on 256 x 256 tiles (dX, dW 128 x 256)
#   (3000, 1544, 2056)  dX on 256 x 256 tiles
#   (2056, 1544, 3080)  dW on 256 x 256 tiles, one split (stored)
#   (12040, 264, 3080)  dW on 256 x 256 tiles, split 5 (fp32 reductions)
#   (3000, 264, 2056)   dW on 128 x 256 tiles, split 4
@pytest.mark.parametrize("shape", [(3000, 776, 776), (3000, 2056, 1544), (3000, 1544, 2056),
                                   (2056, 1544, 3080), (12040, 264, 3080), (3000, 264, 2056)])
def test_wide_tiles_on_ragged_shapes(shape):
    run(*shape, seed=61 + shape[1] % 7)


def test_wide_tiles_fp16_and_fp32_outputs():
    run(3000, 2056, 1544, seed=67, dtype=torch.float16)
    run(3000, 1544, 2056, seed=71, out_f32=True)
