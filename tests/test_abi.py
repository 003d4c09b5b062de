"""The C ABI loads, exports every declared symbol and validates arguments on
the host (no GPU needed: only calls that fail validation are made)."""
import ctypes
import os
import re

import pytest

from gated_delta_rule_133_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "kda.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert {"kda_chunk_fwd", "kda_varlen_fwd", "kda_recurrent_step"} <= set(names)
    lib = _lib.load()
    for n in names:
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, n


def test_status_strings_and_version():
    for st in range(6):
        assert _lib.status_string(st).startswith("KDA_")
    assert "WARN_DOMAIN" in _lib.status_string(_lib.KDA_WARN_DOMAIN)
    assert "UNKNOWN" in _lib.status_string(99)
    assert _lib.load().kda_version() >= 100


P = 256  # a 16-byte aligned fake address: never dereferenced, validation fails first


@pytest.mark.parametrize("args,want", [
    # negative sizes
    ((P, P, P, P, P, None, P, None, -1, 8, 2, 128, 128, 64, 1, 0, None, 0, None), _lib.KDA_ERR_INVALID_ARG),
    ((P, P, P, P, P, None, P, None, 1, -8, 2, 128, 128, 64, 1, 0, None, 0, None), _lib.KDA_ERR_INVALID_ARG),
    ((P, P, P, P, P, None, P, None, 1, 8, 0, 128, 128, 64, 1, 0, None, 0, None), _lib.KDA_ERR_INVALID_ARG),
    # null or misaligned tensors
    ((None, P, P, P, P, None, P, None, 1, 8, 2, 128, 128, 64, 1, 0, None, 0, None), _lib.KDA_ERR_INVALID_ARG),
    ((P + 4, P, P, P, P, None, P, None, 1, 8, 2, 128, 128, 64, 1, 0, None, 0, None), _lib.KDA_ERR_INVALID_ARG),
    ((P, P, P, P, P, P + 8, P, None, 1, 8, 2, 128, 128, 64, 1, 0, None, 0, None), _lib.KDA_ERR_INVALID_ARG),
    # bad dtype code
    ((P, P, P, P, P, None, P, None, 1, 8, 2, 128, 128, 64, 7, 0, None, 0, None), _lib.KDA_ERR_INVALID_ARG),
    ((P, P, P, P, P, None, P, None, 1, 8, 2, 128, 128, 64, 1, 5, None, 0, None), _lib.KDA_ERR_INVALID_ARG),
    # unsupported sizes
    ((P, P, P, P, P, None, P, None, 1, 8, 2, 96, 128, 64, 1, 0, None, 0, None), _lib.KDA_ERR_UNSUPPORTED),
    ((P, P, P, P, P, None, P, None, 1, 8, 2, 128, 256, 64, 1, 0, None, 0, None), _lib.KDA_ERR_UNSUPPORTED),
    ((P, P, P, P, P, None, P, None, 1, 8, 2, 128, 128, 32, 1, 0, None, 0, None), _lib.KDA_ERR_UNSUPPORTED),
])
def test_chunk_fwd_validation(args, want):
    assert _lib.load().kda_chunk_fwd(*args) == want


def test_varlen_validation():
    f = _lib.load().kda_varlen_fwd
    base = [P, P, P, P, P, P, 4, None, P, None, 100, 2, 128, 128, 64, 1, 0, None, 0, None]
    assert f(*base[:6], -1, *base[7:]) == _lib.KDA_ERR_INVALID_ARG          # N < 0
    assert f(*base[:6], 70000, *base[7:]) == _lib.KDA_ERR_INVALID_ARG       # N too large
    assert f(*base[:5], None, *base[6:]) == _lib.KDA_ERR_INVALID_ARG        # no cu_seqlens
    assert f(*base[:5], P + 2, *base[6:]) == _lib.KDA_ERR_INVALID_ARG       # misaligned int32
    assert f(*base[:12], 80, *base[13:]) == _lib.KDA_ERR_UNSUPPORTED         # d_k = 80
    assert f(*base[:6], 0, *base[7:]) == _lib.KDA_ERR_INVALID_ARG           # N = 0 with tokens


def test_recurrent_step_validation():
    f = _lib.load().kda_recurrent_step
    assert f(P, P, P, P, P, P, P, -1, 2, 128, 128, 1, 0, None) == _lib.KDA_ERR_INVALID_ARG
    assert f(P, P, P, P, P, None, P, 3, 2, 128, 128, 1, 0, None) == _lib.KDA_ERR_INVALID_ARG
    assert f(P, P, P, P, P, P, P + 4, 3, 2, 128, 128, 1, 0, None) == _lib.KDA_ERR_INVALID_ARG
    assert f(P, P, P, P + 2, P, P, P, 3, 2, 128, 128, 1, 0, None) == _lib.KDA_ERR_INVALID_ARG  # beta: 4-byte
    assert f(P, P, P, P, P, P, P, 3, 2, 128, 32, 1, 0, None) == _lib.KDA_ERR_UNSUPPORTED
    assert f(P, P, P, P, P, P, P, 3, 2, 128, 128, 1, 9, None) == _lib.KDA_ERR_INVALID_ARG
    assert f(None, None, None, None, None, None, None, 0, 2, 128, 128, 1, 0, None) == _lib.KDA_OK


def test_selftest_timeout_validation():
    f = _lib.load().kda_selftest_timeout
    assert f(0, None) == _lib.KDA_ERR_INVALID_ARG
    assert f(-5, None) == _lib.KDA_ERR_INVALID_ARG
    assert f((1 << 32) + 1, None) == _lib.KDA_ERR_INVALID_ARG


def test_python_binding_rejects_bad_tensors():
    import torch
    import gated_delta_rule_133_b200 as kda
    q = torch.zeros(1, 8, 2, 128)
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd(q, q, q, torch.zeros(1, 8, 2), torch.zeros(1, 8, 2, 64))
    with pytest.raises(ValueError):
        kda.kda_chunk_fwd(q, q, q.to(torch.float64), torch.zeros(1, 8, 2), q)


def test_noalloc_validation():
    """The allocation-free entry point validates like kda_chunk_fwd and rejects,
    on the host, problems whose intermediates do not fit its fixed area."""
    f = _lib.load().kda_chunk_fwd_noalloc
    ok = (P, P, P, P, P, None, P, P, 1, 8, 2, 128, 128, 64, 1, 0, None)
    assert f(*ok[:8], -1, *ok[9:]) == _lib.KDA_ERR_INVALID_ARG
    assert f(None, *ok[1:]) == _lib.KDA_ERR_INVALID_ARG
    assert f(*ok[:11], 96, *ok[12:]) == _lib.KDA_ERR_UNSUPPORTED
    # 20 x 64 (sequence, head) pairs: one chunk of records alone exceeds the 64 MiB area
    assert f(*ok[:8], 20, 8, 64, *ok[11:]) == _lib.KDA_ERR_UNSUPPORTED


def test_mode_validation():
    """Layer variants: unknown mode bits are rejected; a per-head gate array
    needs only 4-byte alignment, a per-channel one 16 bytes."""
    lib = _lib.load()
    base = (P, P, P, P, P, None, P, None, 1, 8, 2, 128, 128, 64, 1, 0)
    ws = (None, 0, None)
    assert lib.kda_chunk_fwd_mode(*base, 32, *ws) == _lib.KDA_ERR_INVALID_ARG
    assert lib.kda_chunk_fwd_mode(*base, -1, *ws) == _lib.KDA_ERR_INVALID_ARG
    assert lib.kda_chunk_fwd_mode(*base, _lib.KDA_MODE_BLOCKS(9), *ws) == _lib.KDA_ERR_INVALID_ARG
    gate4 = base[:4] + (P + 4,) + base[5:]
    assert lib.kda_chunk_fwd_mode(*gate4, _lib.KDA_MODE_NO_ERASE, *ws) == _lib.KDA_ERR_INVALID_ARG
    # 4-byte-aligned per-head gates pass validation: an unsupported head size then decides
    gate4_d96 = gate4[:11] + (96,) + gate4[12:]
    assert lib.kda_chunk_fwd_mode(*gate4_d96, _lib.KDA_MODE_HEAD_GATE, *ws) == _lib.KDA_ERR_UNSUPPORTED
    v = lib.kda_varlen_fwd_mode
    assert v(P, P, P, P, P, P, 1, None, P, None, 8, 2, 128, 128, 64, 1, 0, 32, *ws) == _lib.KDA_ERR_INVALID_ARG
    # the blocked schedule is for dense inputs only
    assert v(P, P, P, P, P, P, 1, None, P, None, 8, 2, 128, 128, 64, 1, 0, _lib.KDA_MODE_BLOCKS(2),
             *ws) == _lib.KDA_ERR_INVALID_ARG
    r = lib.kda_recurrent_step_mode
    assert r(P, P, P, P, P, P, P, 3, 2, 128, 128, 1, 0, 16, None) == _lib.KDA_ERR_INVALID_ARG
    assert r(P, P, P, P, P + 4, P, P, 3, 2, 128, 128, 1, 0, 0, None) == _lib.KDA_ERR_INVALID_ARG
    assert r(P, P, P, P, P + 4, P, P, 3, 2, 96, 128, 1, 0, _lib.KDA_MODE_HEAD_GATE, None) == _lib.KDA_ERR_UNSUPPORTED


def _ws_size(name, *args):
    return _lib.workspace_size(name, *args)


def test_workspace_size_queries():
    """Workspace sizes are a host computation: the tensor-core path needs at
    least one operand record per (chunk, head); the CUDA-core path needs none."""
    B, T, H = 2, 4096, 16
    n = _ws_size("kda_chunk_fwd_workspace_size", B, T, H, 128, 128, 64, _lib.KDA_BF16, 0)
    assert n >= B * (T // 64) * H * 57 * 1024
    assert n % 1024 == 0
    assert _ws_size("kda_chunk_fwd_workspace_size", B, T, H, 128, 128, 64, _lib.KDA_F32, 0) == 0
    assert _ws_size("kda_chunk_fwd_workspace_size", B, T, H, 128, 128, 64, _lib.KDA_BF16,
                    _lib.KDA_MODE_CUDA_CORES) == 0
    assert _ws_size("kda_chunk_fwd_workspace_size", 0, T, H, 128, 128, 64, _lib.KDA_BF16, 0) == 0
    # a ragged tail needs one more chunk of records; d_k = 64 records are smaller
    assert _ws_size("kda_chunk_fwd_workspace_size", B, T + 1, H, 128, 128, 64, _lib.KDA_BF16, 0) > n
    assert _ws_size("kda_chunk_fwd_workspace_size", B, T, H, 64, 64, 64, _lib.KDA_BF16, 0) < n
    nv = _ws_size("kda_varlen_fwd_workspace_size", 8, 65536, 32, 128, 128, 64, _lib.KDA_BF16, 0)
    assert nv >= (65536 // 64) * 32 * 57 * 1024
    # more sequences need room for their ragged last chunks and index arrays
    assert _ws_size("kda_varlen_fwd_workspace_size", 4000, 65536, 32, 128, 128, 64, _lib.KDA_BF16, 0) > nv
    lib = _lib.load()
    out = ctypes.c_size_t(0)
    assert lib.kda_chunk_fwd_workspace_size(B, T, H, 96, 128, 64, 1, 0, ctypes.byref(out)) == _lib.KDA_ERR_UNSUPPORTED
    assert lib.kda_chunk_fwd_workspace_size(-1, T, H, 128, 128, 64, 1, 0, ctypes.byref(out)) == _lib.KDA_ERR_INVALID_ARG
    assert lib.kda_chunk_fwd_workspace_size(B, T, H, 128, 128, 64, 1, 0, None) == _lib.KDA_ERR_INVALID_ARG
    assert lib.kda_varlen_fwd_workspace_size(70000, T, H, 128, 128, 64, 1, 0, ctypes.byref(out)) == \
        _lib.KDA_ERR_INVALID_ARG


def test_undersized_workspace_is_rejected_on_the_host():
    """A workspace smaller than the query's answer, missing or not 256-byte
    aligned returns KDA_ERR_INVALID_ARG before anything is launched."""
    lib = _lib.load()
    B, T, H = 1, 200, 2
    need = _ws_size("kda_chunk_fwd_workspace_size", B, T, H, 128, 128, 64, _lib.KDA_BF16, 0)
    base = (P, P, P, P, P, None, P, None, B, T, H, 128, 128, 64, 1, 0)
    W = 1 << 20   # a 256-byte aligned fake address
    assert lib.kda_chunk_fwd(*base, W, need - 1, None) == _lib.KDA_ERR_INVALID_ARG
    assert lib.kda_chunk_fwd(*base, None, need, None) == _lib.KDA_ERR_INVALID_ARG
    assert lib.kda_chunk_fwd(*base, W + 16, need, None) == _lib.KDA_ERR_INVALID_ARG
    assert lib.kda_chunk_fwd_mode(*base, _lib.KDA_MODE_NO_ERASE, W, 0, None) == _lib.KDA_ERR_INVALID_ARG
    needv = _ws_size("kda_varlen_fwd_workspace_size", 3, T, H, 128, 128, 64, _lib.KDA_BF16, 0)
    v = (P, P, P, P, P, P, 3, None, P, None, T, H, 128, 128, 64, 1, 0)
    assert lib.kda_varlen_fwd(*v, W, needv - 1, None) == _lib.KDA_ERR_INVALID_ARG


def test_backward_and_dplr_workspace_is_checked_on_the_host():
    """The backward and the diagonal-plus-low-rank forward take a caller
    workspace too: the size queries answer on the host, and a workspace that
    is too small, missing or misaligned is refused before any launch."""
    lib = _lib.load()
    B, T, H = 1, 200, 2
    W = 1 << 20   # a 256-byte aligned fake address
    nb = _ws_size("kda_chunk_bwd_workspace_size", B, T, H, 128, 128, 64, _lib.KDA_BF16)
    assert nb >= 4 * H * 64 * 128 * 4   # at least one record per (chunk, head)
    assert _ws_size("kda_chunk_bwd_workspace_size", 0, T, H, 128, 128, 64, _lib.KDA_BF16) == 0
    bwd = (P,) * 14 + (B, T, H, 128, 128, 64, 1)
    assert lib.kda_chunk_bwd(*bwd, W, nb - 1, None) == _lib.KDA_ERR_INVALID_ARG
    assert lib.kda_chunk_bwd(*bwd, None, nb, None) == _lib.KDA_ERR_INVALID_ARG
    assert lib.kda_chunk_bwd(*bwd, W + 16, nb, None) == _lib.KDA_ERR_INVALID_ARG
    nd = _ws_size("kda_dplr_fwd_workspace_size", B, T, H, 128, 128, 64, _lib.KDA_BF16)
    assert nd >= 4 * H * 64 * 128 * 4
    assert _ws_size("kda_dplr_fwd_workspace_size", B, 0, H, 128, 128, 64, _lib.KDA_BF16) == 0
    dp = (P,) * 9 + (B, T, H, 128, 128, 64, 1, 0)
    assert lib.kda_dplr_fwd(*dp, W, nd - 1, None) == _lib.KDA_ERR_INVALID_ARG
    assert lib.kda_dplr_fwd(*dp, None, nd, None) == _lib.KDA_ERR_INVALID_ARG
    ndv = _ws_size("kda_dplr_varlen_fwd_workspace_size", 3, T, H, 128, 128, 64, _lib.KDA_BF16)
    assert ndv > 0
    dv = (P,) * 7 + (3,) + (P,) * 3 + (T, H, 128, 128, 64, 1, 0)
    assert lib.kda_dplr_varlen_fwd(*dv, W, ndv - 1, None) == _lib.KDA_ERR_INVALID_ARG
    out = ctypes.c_size_t(0)
    assert lib.kda_dplr_fwd_workspace_size(B, T, H, 96, 128, 64, 1, ctypes.byref(out)) == _lib.KDA_ERR_UNSUPPORTED
