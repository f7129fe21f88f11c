"""torch-tensor front end of the C ABI: allocates outputs with torch on the inputs'
device, passes raw pointers and the current CUDA stream, checks the status.

PyTorch is plumbing here (device memory and streams).  The arithmetic is in the
CUDA library; there is no CPU path.
"""
from __future__ import annotations

import torch

from . import _lib



def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _check_qkv(*ts: torch.Tensor):
    shape = ts[0].shape
    if len(shape) != 4:
        raise ValueError("expected [B, H, T, d] tensors")
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device (there is no CPU path)")
        if t.dtype != torch.bfloat16:
            raise ValueError("q, k, v, o, dO must be bf16")
        if t.shape != shape:
            raise ValueError("q, k, v, o, dO must have the same shape")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    return shape


def attn_fwd(q, k, v, scale=None, causal=True, o_dtype=torch.bfloat16, precise=False, out=None,
             lse=None):
    """O, LSE = attention forward.  q, k, v: bf16 [B, H, T, d] on one GPU.
    o_dtype: torch.bfloat16 or torch.float32.  precise: split P into hi + lo bf16."""
    B, H, T, d = _check_qkv(q, k, v)
    scale = d ** -0.5 if scale is None else float(scale)
    o = out if out is not None else torch.empty((B, H, T, d), dtype=o_dtype, device=q.device)
    lse = lse if lse is not None else torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    flags = (_lib.OUT_F32 if o.dtype == torch.float32 else 0) | (_lib.PRECISE if precise else 0)
    st = _lib.forge_attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                lse.data_ptr(), B, H, T, d, scale, int(bool(causal)), flags,
                                _stream(q))
    _lib.check(st, "forge_attn_fwd")
    return o, lse


def workspace_bytes(B, H, T, d) -> int:
    return int(_lib.forge_attn_bwd_workspace_size(B, H, T, d))


def attn_bwd(q, k, v, o, dO, lse, scale=None, causal=True, grad_dtype=torch.bfloat16,
             precise=False, workspace=None, out=None):
    """dQ, dK, dV = attention backward (o and lse from attn_fwd; o bf16 or fp32).
    grad_dtype: torch.bfloat16 or torch.float32.  precise: split P and dS into hi + lo."""
    o_f32 = o.dtype == torch.float32
    B, H, T, d = _check_qkv(q, k, v, dO, *(() if o_f32 else (o,)))
    if o.shape != q.shape or not o.is_contiguous():
        raise ValueError("o must be contiguous with the shape of q")
    scale = d ** -0.5 if scale is None else float(scale)
    n = workspace_bytes(B, H, T, d)
    if workspace is None:
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    if out is None:
        out = tuple(torch.empty((B, H, T, d), dtype=grad_dtype, device=q.device) for _ in range(3))
    dq, dk, dv = out
    flags = ((_lib.OUT_F32 if grad_dtype == torch.float32 else 0)
             | (_lib.O_IN_F32 if o_f32 else 0) | (_lib.PRECISE if precise else 0))
    st = _lib.forge_attn_bwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                dO.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                dv.data_ptr(), workspace.data_ptr(), workspace.numel(), B, H, T,
                                d, scale, int(bool(causal)), flags, _stream(q))
    _lib.check(st, "forge_attn_bwd")
    return dq, dk, dv


def check_device_error(device=None):
    """Synchronise the current stream and raise if a bounded device wait ran out."""
    s = torch.cuda.current_stream(device).cuda_stream
    st, detail = _lib.forge_attn_check_device_error(s)
    if st != _lib.OK:
        raise _lib.ForgeAttnError(st, f"device error word 0x{detail:08x}")
