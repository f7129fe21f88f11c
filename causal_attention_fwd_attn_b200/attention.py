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

_GRAD_DTYPES = (torch.bfloat16, torch.float32)


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
    if not isinstance(q, torch.Tensor) or q.dim() != 4:
        raise ValueError("q must be a [B, H, T, d] tensor")
    if not q.is_cuda:
        raise ValueError("tensors must be on a CUDA device (there is no CPU path)")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_tensor(t, name, q.shape, (torch.bfloat16,), q.device)
    return tuple(q.shape)


def attn_fwd(q, k, v, scale=None, causal=True, o_dtype=torch.bfloat16, precise=False, out=None,
             lse=None):
    """O, LSE = attention forward.  q, k, v: bf16 [B, H, T, d] on one GPU.
    o_dtype: torch.bfloat16 or torch.float32 (ignored when `out` is given: its dtype
    decides).  precise: split P into hi + lo bf16.  lse: fp32 [B, H, T]."""
    B, H, T, d = _check_qkv(q, k, v)
    dev = q.device
    scale = d ** -0.5 if scale is None else float(scale)
    if out is None:
        if o_dtype not in _GRAD_DTYPES:
            raise ValueError(f"o_dtype must be one of {_GRAD_DTYPES}")
        out = torch.empty((B, H, T, d), dtype=o_dtype, device=dev)
    o = _check_tensor(out, "out", (B, H, T, d), _GRAD_DTYPES, dev)
    if lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    _check_tensor(lse, "lse", (B, H, T), (torch.float32,), dev)
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
    grad_dtype: torch.bfloat16 or torch.float32 (ignored when `out` is given: the
    three output tensors share one dtype, which decides).  precise: split P and dS
    into hi + lo.  workspace: a uint8 tensor of at least workspace_bytes() bytes."""
    B, H, T, d = _check_qkv(q, k, v)
    dev = q.device
    _check_tensor(dO, "dO", (B, H, T, d), (torch.bfloat16,), dev)
    _check_tensor(o, "o", (B, H, T, d), _GRAD_DTYPES, dev)
    _check_tensor(lse, "lse", (B, H, T), (torch.float32,), dev)
    scale = d ** -0.5 if scale is None else float(scale)
    n = workspace_bytes(B, H, T, d)
    if workspace is None:
        workspace = torch.empty(n, dtype=torch.uint8, device=dev)
    _check_tensor(workspace, "workspace", tuple(workspace.shape), (torch.uint8,), dev)
    if workspace.numel() < n:
        raise ValueError(f"workspace has {workspace.numel()} bytes, needs {n}")
    if out is None:
        if grad_dtype not in _GRAD_DTYPES:
            raise ValueError(f"grad_dtype must be one of {_GRAD_DTYPES}")
        out = tuple(torch.empty((B, H, T, d), dtype=grad_dtype, device=dev) for _ in range(3))
    if len(out) != 3:
        raise ValueError("out must be (dq, dk, dv)")
    dq, dk, dv = (_check_tensor(t, name, (B, H, T, d), _GRAD_DTYPES, dev)
                  for name, t in zip(("dq", "dk", "dv"), out))
    if not dq.dtype == dk.dtype == dv.dtype:
        raise ValueError("dq, dk, dv must share one dtype")
    flags = ((_lib.OUT_F32 if dq.dtype == torch.float32 else 0)
             | (_lib.O_IN_F32 if o.dtype == torch.float32 else 0)
             | (_lib.PRECISE if precise else 0))
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
