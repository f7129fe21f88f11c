"""ctypes binding of libforge_attn.so: the C ABI of include/forge_attn.h and
include/forge_attn_testing.h under the same names.

Argument marshalling only.  Every step of the operation runs in the library's
CUDA kernels; nothing here computes, and there is no fallback: if the shared
library is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

from . import build as _build

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_MISALIGNED = 3
ERR_CUDA = 4
ERR_TIMEOUT = 5
ERR_WORKSPACE = 6
# option bits of the _ex entry points
OUT_F32 = 1
O_IN_F32 = 2
PRECISE = 4
FP16 = 8

PROBE_SS_KK = 0
PROBE_SS_KMN = 1
PROBE_TS_KMN = 2
PROBE_SS_MNMN = 3

EXPORTED = [
    "forge_attn_fwd", "forge_attn_fwd_ex", "forge_attn_bwd_workspace_size", "forge_attn_bwd",
    "forge_attn_bwd_ex", "forge_attn_bwd_preprocess", "forge_attn_bwd_dkdv",
    "forge_attn_bwd_dq_convert", "forge_attn_bwd_dq_convert_ex", "forge_attn_status_string",
    "forge_attn_check_device_error", "forge_attn_version", "forge_probe_mma", "forge_probe_wait_timeout",
    "forge_attn_bwd_noalloc", "forge_adamw_workspace_size", "forge_adamw_step",
    "forge_linear_fwd", "forge_linear_bwd_dx", "forge_linear_bwd_dw", "forge_linear_split_k",
    "forge_attn_bf16_to_fp16",
]

ADAMW_MAX_TENSORS_PER_LAUNCH = 256


class AdamWTensor(ctypes.Structure):
    """forge_adamw_tensor of include/forge_adamw.h (device pointers and a size)."""
    _fields_ = [("param", ctypes.c_void_p), ("grad", ctypes.c_void_p),
                ("exp_avg", ctypes.c_void_p), ("exp_avg_sq", ctypes.c_void_p),
                ("n", ctypes.c_longlong), ("decay", ctypes.c_int)]


_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_sz = ctypes.c_size_t

_SIGNATURES = {
    "forge_attn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp]),
    "forge_attn_fwd_ex": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _i, _vp]),
    "forge_attn_bwd_workspace_size": (_sz, [_i, _i, _i, _i]),
    "forge_attn_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _i, _i, _i,
                            _i, _f, _i, _vp]),
    "forge_attn_bwd_ex": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _i, _i,
                               _i, _i, _f, _i, _i, _vp]),
    "forge_attn_bwd_preprocess": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "forge_attn_bwd_dkdv": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i,
                                 _i, _vp]),
    "forge_attn_bwd_dq_convert": (_i, [_vp, _vp, _i, _i, _i, _i, _vp]),
    "forge_attn_bwd_dq_convert_ex": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "forge_attn_status_string": (ctypes.c_char_p, [_i]),
    "forge_attn_check_device_error": (_i, [_vp, ctypes.POINTER(ctypes.c_uint)]),
    "forge_attn_version": (_i, []),
    "forge_probe_mma": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp]),
    "forge_probe_wait_timeout": (_i, [ctypes.c_ulonglong, _vp]),
    "forge_attn_bwd_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                    _f, _i, _vp]),
    "forge_adamw_workspace_size": (_sz, [_i]),
    "forge_linear_fwd": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp]),
    "forge_linear_bwd_dx": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp]),
    "forge_linear_bwd_dw": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]),
    "forge_linear_split_k": (_i, [_i, _i, _i]),
    "forge_attn_bf16_to_fp16": (_i, [_vp, _vp, ctypes.c_longlong, _vp, _vp]),
    "forge_adamw_step": (_i, [ctypes.POINTER(AdamWTensor), _i, _f, _f, _f, _f, _f, _i, _f, _vp,
                              _vp, _sz, _vp]),
}

_lib = None


class ForgeAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def library_path() -> str:
    return _build.LIBRARY


def load(path: str | None = None):
    """Load (once) and return the ctypes handle.  Raises if the library is missing."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or library_path()
    if not os.path.exists(p):
        raise RuntimeError(
            f"the CUDA library {p} is not built; run python -m causal_attention_fwd_attn_b200.build")
    lib = ctypes.CDLL(p)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().forge_attn_status_string(int(status)).decode()


def check(status: int, where: str) -> None:
    if status != OK:
        raise ForgeAttnError(status, where)


# -- the ABI under its own names ---------------------------------------------------
def forge_attn_fwd(q, k, v, o, lse, B, H, T, d, scale, causal, stream):
    return load().forge_attn_fwd(q, k, v, o, lse, B, H, T, d, scale, causal, stream)


def forge_attn_fwd_ex(q, k, v, o, lse, B, H, T, d, scale, causal, flags, stream):
    return load().forge_attn_fwd_ex(q, k, v, o, lse, B, H, T, d, scale, causal, flags, stream)


def forge_attn_bwd_workspace_size(B, H, T, d):
    return load().forge_attn_bwd_workspace_size(B, H, T, d)


def forge_attn_bwd(q, k, v, o, dO, lse, dq, dk, dv, workspace, workspace_bytes, B, H, T, d,
                   scale, causal, stream):
    return load().forge_attn_bwd(q, k, v, o, dO, lse, dq, dk, dv, workspace, workspace_bytes,
                                 B, H, T, d, scale, causal, stream)


def forge_attn_bwd_ex(q, k, v, o, dO, lse, dq, dk, dv, workspace, workspace_bytes, B, H, T, d,
                      scale, causal, flags, stream):
    return load().forge_attn_bwd_ex(q, k, v, o, dO, lse, dq, dk, dv, workspace,
                                    workspace_bytes, B, H, T, d, scale, causal, flags, stream)


def forge_attn_bwd_preprocess(o, dO, lse, rowstats, dq_accum, B, H, T, d, flags, stream):
    return load().forge_attn_bwd_preprocess(o, dO, lse, rowstats, dq_accum, B, H, T, d, flags,
                                            stream)


def forge_attn_bwd_dkdv(q, k, v, dO, rowstats, dq_accum, dk, dv, B, H, T, d, scale, causal,
                        flags, stream):
    return load().forge_attn_bwd_dkdv(q, k, v, dO, rowstats, dq_accum, dk, dv, B, H, T, d,
                                      scale, causal, flags, stream)


def rowstats_bytes(B, H, T):
    """Bytes of the padded row statistics at the start of the backward workspace."""
    t_pad = -(-T // 128) * 128
    return -(-(2 * B * H * t_pad * 4) // 256) * 256


def forge_attn_bwd_dq_convert(dq_accum, dq, B, H, T, d, stream):
    return load().forge_attn_bwd_dq_convert(dq_accum, dq, B, H, T, d, stream)


def forge_attn_bwd_dq_convert_ex(dq_accum, dq, B, H, T, d, flags, stream):
    return load().forge_attn_bwd_dq_convert_ex(dq_accum, dq, B, H, T, d, flags, stream)


def forge_attn_bwd_noalloc(q, k, v, o, dO, lse, dq, dk, dv, B, H, T, d, scale, causal, stream):
    return load().forge_attn_bwd_noalloc(q, k, v, o, dO, lse, dq, dk, dv, B, H, T, d, scale,
                                         causal, stream)


NOALLOC_SCRATCH_BYTES = 64 << 20


def forge_adamw_workspace_size(n_tensors):
    return load().forge_adamw_workspace_size(n_tensors)


def forge_adamw_step(tensors, lr, beta1, beta2, eps, weight_decay, step, max_norm,
                     grad_norm_out, workspace, workspace_bytes, stream):
    """tensors: a sequence of (param, grad, exp_avg, exp_avg_sq, n, decay) tuples of device
    addresses and sizes, or AdamWTensor values."""
    arr = (AdamWTensor * max(1, len(tensors)))()
    for i, t in enumerate(tensors):
        arr[i] = t if isinstance(t, AdamWTensor) else AdamWTensor(*t)
    return load().forge_adamw_step(arr, len(tensors), lr, beta1, beta2, eps, weight_decay, step,
                                   max_norm, grad_norm_out, workspace, workspace_bytes, stream)


def forge_linear_fwd(x, w, y, tokens, in_features, out_features, flags, stream):
    return load().forge_linear_fwd(x, w, y, tokens, in_features, out_features, flags, stream)


def forge_linear_bwd_dx(dy, w, dx, tokens, in_features, out_features, flags, stream):
    return load().forge_linear_bwd_dx(dy, w, dx, tokens, in_features, out_features, flags,
                                      stream)


def forge_linear_bwd_dw(dy, x, dw, tokens, in_features, out_features, split_k, accumulate,
                        flags, stream):
    return load().forge_linear_bwd_dw(dy, x, dw, tokens, in_features, out_features, split_k,
                                      accumulate, flags, stream)


def forge_linear_split_k(tokens, in_features, out_features):
    return load().forge_linear_split_k(tokens, in_features, out_features)


def forge_attn_bf16_to_fp16(src, dst, n, overflow, stream):
    return load().forge_attn_bf16_to_fp16(src, dst, n, overflow, stream)


def forge_attn_check_device_error(stream):
    detail = ctypes.c_uint(0)
    st = load().forge_attn_check_device_error(stream, ctypes.byref(detail))
    return st, detail.value


def forge_attn_version():
    return load().forge_attn_version()


def forge_probe_mma(a, b, d_out, N, K, mode, stream):
    return load().forge_probe_mma(a, b, d_out, N, K, mode, stream)


def forge_probe_wait_timeout(limit_ns, stream):
    return load().forge_probe_wait_timeout(limit_ns, stream)
