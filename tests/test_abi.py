"""The C ABI library: it loads, exports every function the headers declare, and
rejects bad arguments on the host before any launch (CPU only: no call here
reaches the GPU)."""
import ctypes
import os
import re

import pytest

from causal_attention_fwd_attn_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h)
           for h in ("forge_attn.h", "forge_attn_testing.h", "forge_adamw.h", "forge_linear.h")]


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    names = []
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_headers_declare_the_binding():
    assert declared_functions() == sorted(_lib.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_version_and_status_strings(lib):
    assert _lib.forge_attn_version() == 100
    for code in range(7):
        assert _lib.status_string(code)
    assert "unknown" in _lib.status_string(99)


def _up256(x):
    return (x + 255) // 256 * 256


def test_workspace_size(lib):
    # padded row statistics (2 x B*H x 128*ceil(T/128) fp32), then the fp32 dQ accumulator
    n = _lib.forge_attn_bwd_workspace_size(1, 2, 128, 64)
    assert n == _up256(2 * 2 * 128 * 4) + _up256(2 * 128 * 64 * 4)
    assert _lib.forge_attn_bwd_workspace_size(1, 1, 1, 96) == 0
    assert _lib.forge_attn_bwd_workspace_size(0, 1, 1, 64) == 0
    # ragged T: the statistics are padded to whole tiles, both parts 256-byte aligned
    n = _lib.forge_attn_bwd_workspace_size(1, 1, 7, 64)
    assert n == _up256(2 * 128 * 4) + _up256(7 * 64 * 4)
    assert _lib.rowstats_bytes(3, 5, 200) == _up256(2 * 15 * 256 * 4)


P = 4096  # a 16-byte aligned fake address; never dereferenced (rejected first)


@pytest.mark.parametrize("args,want", [
    ((0, P, P, P, P, 1, 1, 8, 64, 0.1, 1), _lib.ERR_INVALID_ARG),      # null q
    ((P, P, P, P, 0, 1, 1, 8, 64, 0.1, 1), _lib.ERR_INVALID_ARG),      # null lse
    ((P, P, P, P, P, 0, 1, 8, 64, 0.1, 1), _lib.ERR_INVALID_ARG),      # B = 0
    ((P, P, P, P, P, 1, 1, 0, 64, 0.1, 1), _lib.ERR_INVALID_ARG),      # T = 0
    ((P, P, P, P, P, 1, 1, 8, 96, 0.1, 1), _lib.ERR_UNSUPPORTED),      # d = 96
    ((P, P, P, P, P, 1, 1, 8, 32, 0.1, 1), _lib.ERR_UNSUPPORTED),      # d = 32
    ((P, P, P, P, P, 1, 1, 8, 64, float("nan"), 1), _lib.ERR_INVALID_ARG),
    ((P, P, P, P, P, 1, 1, 8, 64, float("inf"), 1), _lib.ERR_INVALID_ARG),
    ((P, P, P, P, P, 1, 1, 8, 64, 0.1, 2), _lib.ERR_INVALID_ARG),      # causal flag
    ((P + 8, P, P, P, P, 1, 1, 8, 64, 0.1, 1), _lib.ERR_MISALIGNED),   # q not 16-B aligned
    ((P, P, P, P + 2, P, 1, 1, 8, 64, 0.1, 1), _lib.ERR_MISALIGNED),   # o
    ((P, P, P, P, P + 2, 1, 1, 8, 64, 0.1, 1), _lib.ERR_MISALIGNED),   # lse not 4-B aligned
    ((P, P, P, P, P, 1 << 16, 1 << 10, 64, 64, 0.1, 1), _lib.ERR_UNSUPPORTED),  # too large
])
def test_fwd_rejects_bad_arguments(lib, args, want):
    assert _lib.forge_attn_fwd(*args, None) == want


def test_fwd_rejects_unknown_flags(lib):
    assert _lib.forge_attn_fwd_ex(P, P, P, P, P, 1, 1, 8, 64, 0.1, 1, 16, None) == \
        _lib.ERR_INVALID_ARG
    # fp16 operands and the bf16 hi + lo split do not combine
    assert _lib.forge_attn_fwd_ex(P, P, P, P, P, 1, 1, 8, 64, 0.1, 1,
                                  _lib.FP16 | _lib.PRECISE, None) == _lib.ERR_UNSUPPORTED
    # O_IN_F32 means nothing to the forward
    assert _lib.forge_attn_fwd_ex(P, P, P, P, P, 1, 1, 8, 64, 0.1, 1, _lib.O_IN_F32, None) == \
        _lib.ERR_INVALID_ARG


def test_bwd_rejects_bad_arguments(lib):
    ws = _lib.forge_attn_bwd_workspace_size(1, 1, 8, 64)
    good = [P] * 10 + [ws, 1, 1, 8, 64, 0.1, 1]
    assert _lib.forge_attn_bwd(*[0] + good[1:], None) == _lib.ERR_INVALID_ARG
    bad = list(good)
    bad[10] = ws - 1
    assert _lib.forge_attn_bwd(*bad, None) == _lib.ERR_WORKSPACE
    bad = list(good)
    bad[9] = 0
    assert _lib.forge_attn_bwd(*bad, None) == _lib.ERR_WORKSPACE
    bad = list(good)
    bad[9] = P + 16  # workspace must be 256-byte aligned
    assert _lib.forge_attn_bwd(*bad, None) == _lib.ERR_MISALIGNED
    bad = list(good)
    bad[14] = 80
    assert _lib.forge_attn_bwd(*bad, None) == _lib.ERR_UNSUPPORTED
    assert _lib.forge_attn_bwd_ex(*good, 16, None) == _lib.ERR_INVALID_ARG
    assert _lib.forge_attn_bwd_ex(*good, _lib.FP16 | _lib.PRECISE, None) == _lib.ERR_UNSUPPORTED


def test_stage_entry_points_reject_bad_arguments(lib):
    assert _lib.forge_attn_bwd_preprocess(0, P, P, P, P, 1, 1, 8, 64, 0, None) == \
        _lib.ERR_INVALID_ARG
    assert _lib.forge_attn_bwd_preprocess(P, P, P, P, P + 4, 1, 1, 8, 64, 0, None) == \
        _lib.ERR_MISALIGNED
    assert _lib.forge_attn_bwd_preprocess(P, P, P, P + 8, P, 1, 1, 8, 64, 0, None) == \
        _lib.ERR_MISALIGNED  # row statistics must be 16-byte aligned
    assert _lib.forge_attn_bwd_preprocess(P, P, P, P, P, 1, 1, 8, 64, _lib.PRECISE, None) == \
        _lib.ERR_INVALID_ARG
    assert _lib.forge_attn_bwd_dkdv(P, P, P, P, P, 0, P, P, 1, 1, 8, 64, 0.1, 1, 0, None) == \
        _lib.ERR_INVALID_ARG
    assert _lib.forge_attn_bwd_dq_convert(P, P, 1, 1, 8, 48, None) == _lib.ERR_UNSUPPORTED
    assert _lib.forge_attn_bwd_dq_convert_ex(P, P, 1, 1, 8, 64, _lib.PRECISE, None) == \
        _lib.ERR_INVALID_ARG
    assert _lib.forge_attn_bwd_dkdv(P, P, P, P, P, P, P, P, 1, 1, 8, 64, 0.1, 1,
                                    _lib.FP16 | _lib.PRECISE, None) == _lib.ERR_UNSUPPORTED
    assert _lib.forge_probe_mma(P, P, P, 96, 64, 0, None) == _lib.ERR_INVALID_ARG
    assert _lib.forge_probe_mma(P, P, P, 64, 64, 9, None) == _lib.ERR_INVALID_ARG


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="not built"):
        _lib.load(os.path.join(tmp_path, "libforge_attn.so"))


def test_library_has_no_oracle_dependency(lib):
    # the product library and the oracle share no code: no oracle symbol inside
    names = open(_lib.library_path(), "rb").read()
    assert b"oracle_attn" not in names
    assert ctypes.CDLL(_lib.library_path())  # loads without a GPU


def test_adamw_rejects_bad_arguments(lib):
    ws_n = _lib.forge_adamw_workspace_size(1)
    assert ws_n >= 16 and _lib.forge_adamw_workspace_size(0) == 0
    ok = [(P, P + 256, P + 512, P + 768, 8, 1)]
    common = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, max_norm=1.0,
                  grad_norm_out=None, workspace=P + 4096, stream=None)
    assert _lib.forge_adamw_step(ok, step=0, workspace_bytes=ws_n, **common) == \
        _lib.ERR_INVALID_ARG
    assert _lib.forge_adamw_step([(P + 4, P, P, P, 8, 1)], step=1, workspace_bytes=ws_n,
                                 **common) == _lib.ERR_MISALIGNED
    assert _lib.forge_adamw_step(ok, step=1, workspace_bytes=ws_n - 1, **common) == \
        _lib.ERR_WORKSPACE
    assert _lib.forge_adamw_step([(P, P, P, P, 0, 1)], step=1, workspace_bytes=ws_n,
                                 **common) == _lib.ERR_INVALID_ARG
    assert _lib.forge_adamw_step(ok, step=1, workspace_bytes=ws_n,
                                 **dict(common, beta2=1.0)) == _lib.ERR_INVALID_ARG
    assert _lib.forge_adamw_step([], step=1, workspace_bytes=ws_n, **common) == \
        _lib.ERR_INVALID_ARG


def test_linear_rejects_bad_arguments(lib):
    assert _lib.forge_linear_fwd(0, P, P, 64, 64, 64, 0, None) == _lib.ERR_INVALID_ARG
    assert _lib.forge_linear_fwd(P, P, P, 64, 60, 64, 0, None) == _lib.ERR_UNSUPPORTED
    assert _lib.forge_linear_fwd(P, P, P, 0, 64, 64, 0, None) == _lib.ERR_INVALID_ARG
    assert _lib.forge_linear_fwd(P, P, P + 8, 64, 64, 64, 0, None) == _lib.ERR_MISALIGNED
    assert _lib.forge_linear_fwd(P, P, P, 64, 64, 64, _lib.PRECISE, None) == _lib.ERR_INVALID_ARG
    assert _lib.forge_linear_bwd_dx(P, P, P, 64, 64, 12, 0, None) == _lib.ERR_UNSUPPORTED
    assert _lib.forge_linear_bwd_dw(P, P, P, 64, 64, 64, -1, 0, 0, None) == _lib.ERR_INVALID_ARG
    assert _lib.forge_linear_bwd_dw(P, P, P, 64, 64, 64, 1, 2, 0, None) == _lib.ERR_INVALID_ARG
    assert _lib.forge_linear_bwd_dw(P, P, P, 64, 64, 64, 1, 0, _lib.OUT_F32, None) == \
        _lib.ERR_INVALID_ARG
    assert _lib.forge_linear_split_k(8192, 768, 3072) >= 1
    assert _lib.forge_linear_split_k(8, 8, 0) == 0


def test_bf16_to_fp16_rejects_bad_arguments(lib):
    # all checked before any launch (no GPU needed); n = 0 is a no-op
    Q = P + (1 << 20)
    assert _lib.forge_attn_bf16_to_fp16(P, Q, 0, None, None) == _lib.OK
    assert _lib.forge_attn_bf16_to_fp16(P, Q, -1, None, None) == _lib.ERR_INVALID_ARG
    assert _lib.forge_attn_bf16_to_fp16(0, Q, 8, None, None) == _lib.ERR_INVALID_ARG
    assert _lib.forge_attn_bf16_to_fp16(P, 0, 8, None, None) == _lib.ERR_INVALID_ARG
    assert _lib.forge_attn_bf16_to_fp16(P + 2, Q, 8, None, None) == _lib.ERR_MISALIGNED
    assert _lib.forge_attn_bf16_to_fp16(P, Q + 8, 8, None, None) == _lib.ERR_MISALIGNED
    assert _lib.forge_attn_bf16_to_fp16(P, Q, 8, Q + 2, None) == _lib.ERR_MISALIGNED
    # overlapping source and destination
    assert _lib.forge_attn_bf16_to_fp16(P, P + 16, 64, None, None) == _lib.ERR_INVALID_ARG
    assert _lib.forge_attn_bf16_to_fp16(P + 16, P, 64, None, None) == _lib.ERR_INVALID_ARG
