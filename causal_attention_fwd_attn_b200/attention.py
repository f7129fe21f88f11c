"""torch-tensor front end of the C ABI: allocates outputs with torch on the inputs'
device, passes raw pointers and the current CUDA stream, checks the status.

PyTorch is plumbing here (device memory and streams).  The arithmetic is in the
CUDA library; there is no CPU path.  The C ABI sees raw pointers only, so every
tensor handed to it (inputs, caller-supplied outputs and workspace) is checked here
for device, dtype, shape and layout first: a wrong buffer raises ValueError instead
of being written past its end.
"""
from __future__ import annotations

import torch

from . import _lib

_IN_DTYPES = (torch.bfloat16, torch.float16)
_GRAD_DTYPES = (torch.bfloat16, torch.float32)


def _out_dtypes(in_dtype):
    """Output dtypes for inputs of `in_dtype`: that 16-bit type, or fp32."""
    return (in_dtype, torch.float32)


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _check_tensor(t, name: str, shape, dtypes, device: torch.device) -> torch.Tensor:
    """`t` must be a contiguous tensor of `shape`, one of `dtypes`, on `device`."""
    if not isinstance(t, torch.Tensor):
        raise ValueError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}, expected one of {tuple(dtypes)}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _check_qkv(q, k, v):
    """q, k, v: one shape, one 16-bit dtype (bf16, or fp16 for the fp16-operand kernels)."""
    if not isinstance(q, torch.Tensor) or q.dim() != 4:
        raise ValueError("q must be a [B, H, T, d] tensor")
    if not q.is_cuda:
        raise ValueError("tensors must be on a CUDA device (there is no CPU path)")
    _check_tensor(q, "q", q.shape, _IN_DTYPES, q.device)
    for name, t in (("k", k), ("v", v)):
        _check_tensor(t, name, q.shape, (q.dtype,), q.device)
    return tuple(q.shape)


def _fp16_flag(q):
    return _lib.FP16 if q.dtype == torch.float16 else 0


def to_fp16(x: torch.Tensor) -> torch.Tensor:
    """fp16 copy of a bf16 CUDA tensor through the library's conversion (round to nearest
    even: exact for magnitudes in [2^-14, 65504]), for the fp16-operand kernels, whose
    P and dS keep 11 significant bits.  Raises ValueError if a value lies beyond fp16's
    range (this reads the overflow count, so it synchronises the stream)."""
    if not isinstance(x, torch.Tensor) or not x.is_cuda:
        raise ValueError("x must be a CUDA tensor (there is no CPU path)")
    _check_tensor(x, "x", tuple(x.shape), (torch.bfloat16,), x.device)
    y = torch.empty_like(x, dtype=torch.float16)
    over = torch.zeros(1, dtype=torch.int32, device=x.device)
    _lib.check(_lib.forge_attn_bf16_to_fp16(x.data_ptr(), y.data_ptr(), x.numel(),
                                            over.data_ptr(), _stream(x)), "forge_attn_bf16_to_fp16")
    n = int(over.item())
    if n:
        raise ValueError(f"{n} values beyond fp16's range (65504)")
    return y


def attn_fwd(q, k, v, scale=None, causal=True, o_dtype=None, precise=False, out=None,
             lse=None):
    """O, LSE = attention forward.  q, k, v: bf16 [B, H, T, d] on one GPU (or all fp16:
    the fp16-operand kernels).  o_dtype: the inputs' 16-bit type (default) or
    torch.float32 (ignored when `out` is given: its dtype decides).  precise: split P
    into hi + lo bf16 (bf16 inputs only).  lse: fp32 [B, H, T]."""
    B, H, T, d = _check_qkv(q, k, v)
    dev = q.device
    outs = _out_dtypes(q.dtype)
    scale = d ** -0.5 if scale is None else float(scale)
    if out is None:
        o_dtype = q.dtype if o_dtype is None else o_dtype
        if o_dtype not in outs:
            raise ValueError(f"o_dtype must be one of {outs}")
        out = torch.empty((B, H, T, d), dtype=o_dtype, device=dev)
    o = _check_tensor(out, "out", (B, H, T, d), outs, dev)
    if lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    _check_tensor(lse, "lse", (B, H, T), (torch.float32,), dev)
    flags = ((_lib.OUT_F32 if o.dtype == torch.float32 else 0) | (_lib.PRECISE if precise else 0)
             | _fp16_flag(q))
    st = _lib.forge_attn_fwd_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                lse.data_ptr(), B, H, T, d, scale, int(bool(causal)), flags,
                                _stream(q))
    _lib.check(st, "forge_attn_fwd")
    return o, lse


def workspace_bytes(B, H, T, d) -> int:
    return int(_lib.forge_attn_bwd_workspace_size(B, H, T, d))


def attn_bwd(q, k, v, o, dO, lse, scale=None, causal=True, grad_dtype=None,
             precise=False, workspace=None, out=None):
    """dQ, dK, dV = attention backward (o and lse from attn_fwd; o in the inputs' 16-bit
    type or fp32; dO in the inputs' type).  grad_dtype: the inputs' 16-bit type
    (default) or torch.float32 (ignored when `out` is given: the three output tensors
    share one dtype, which decides).  precise: split P and dS into hi + lo (bf16 inputs
    only).  workspace: a uint8 tensor of at least workspace_bytes() bytes."""
    B, H, T, d = _check_qkv(q, k, v)
    dev = q.device
    outs = _out_dtypes(q.dtype)
    _check_tensor(dO, "dO", (B, H, T, d), (q.dtype,), dev)
    _check_tensor(o, "o", (B, H, T, d), outs, dev)
    _check_tensor(lse, "lse", (B, H, T), (torch.float32,), dev)
    scale = d ** -0.5 if scale is None else float(scale)
    n = workspace_bytes(B, H, T, d)
    if workspace is None:
        workspace = torch.empty(n, dtype=torch.uint8, device=dev)
    _check_tensor(workspace, "workspace", tuple(workspace.shape), (torch.uint8,), dev)
    if workspace.numel() < n:
        raise ValueError(f"workspace has {workspace.numel()} bytes, needs {n}")
    if out is None:
        grad_dtype = q.dtype if grad_dtype is None else grad_dtype
        if grad_dtype not in outs:
            raise ValueError(f"grad_dtype must be one of {outs}")
        out = tuple(torch.empty((B, H, T, d), dtype=grad_dtype, device=dev) for _ in range(3))
    if len(out) != 3:
        raise ValueError("out must be (dq, dk, dv)")
    dq, dk, dv = (_check_tensor(t, name, (B, H, T, d), outs, dev)
                  for name, t in zip(("dq", "dk", "dv"), out))
    if not dq.dtype == dk.dtype == dv.dtype:
        raise ValueError("dq, dk, dv must share one dtype")
    flags = ((_lib.OUT_F32 if dq.dtype == torch.float32 else 0)
             | (_lib.O_IN_F32 if o.dtype == torch.float32 else 0)
             | (_lib.PRECISE if precise else 0) | _fp16_flag(q))
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
