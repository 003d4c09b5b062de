"""ctypes loader for the in-tree CUDA library ``libkda.so`` (declared in include/kda.h).

There is no fallback: if the library is missing or fails to load, every call
raises.  Build it with ``python -m gated_delta_rule_133_b200.build`` (or
``__graft_entry__.build()``).
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkda.so")

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_CUDA, KDA_ERR_TIMEOUT, KDA_WARN_DOMAIN = range(6)
KDA_F32, KDA_BF16 = 0, 1
KDA_MODE_HEAD_GATE, KDA_MODE_NO_ERASE, KDA_MODE_NORM_QK, KDA_MODE_GATE_LOGITS = 1, 2, 4, 8
KDA_MODE_CUDA_CORES = 16


def KDA_MODE_BLOCKS(n: int) -> int:
    return n << 8


# Every symbol include/kda.h declares, with its ctypes signature.
_P = ctypes.c_void_p
_I = ctypes.c_int
_Z = ctypes.c_size_t
_ZP = ctypes.POINTER(ctypes.c_size_t)
SIGNATURES = {
    "kda_chunk_fwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _Z, _P]),
    "kda_chunk_fwd_workspace_size": (_I, [_I, _I, _I, _I, _I, _I, _I, _I, _ZP]),
    "kda_chunk_fwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P]),
    "kda_varlen_fwd": (_I, [_P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _Z, _P]),
    "kda_varlen_fwd_workspace_size": (_I, [_I, _I, _I, _I, _I, _I, _I, _I, _ZP]),
    "kda_recurrent_step": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    "kda_chunk_fwd_mode": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P, _Z, _P]),
    "kda_varlen_fwd_mode": (_I, [_P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _Z,
                                 _P]),
    "kda_recurrent_step_mode": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P]),
    "kda_chunk_bwd": (_I, [_P] * 14 + [_I, _I, _I, _I, _I, _I, _I, _P, _Z, _P]),
    "kda_chunk_bwd_workspace_size": (_I, [_I, _I, _I, _I, _I, _I, _I, _ZP]),
    "kda_varlen_bwd": (_I, [_P] * 6 + [_I] + [_P] * 9 + [_I, _I, _I, _I, _I, _I, _P, _Z, _P]),
    "kda_varlen_bwd_workspace_size": (_I, [_I, _I, _I, _I, _I, _I, _I, _ZP]),
    "kda_dplr_fwd": (_I, [_P] * 9 + [_I] * 8 + [_P, _Z, _P]),
    "kda_dplr_fwd_workspace_size": (_I, [_I] * 7 + [_ZP]),
    "kda_dplr_varlen_fwd": (_I, [_P] * 7 + [_I] + [_P] * 3 + [_I] * 7 + [_P, _Z, _P]),
    "kda_dplr_varlen_fwd_workspace_size": (_I, [_I] * 7 + [_ZP]),
    "kda_check": (_I, [_P]),
    "kda_selftest_timeout": (_I, [ctypes.c_longlong, _P]),
    "kda_status_string": (ctypes.c_char_p, [_I]),
    "kda_version": (_I, []),
}

_lib = None


class KdaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def load():
    """Load libkda.so once; raises if it is not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run python -m gated_delta_rule_133_b200.build")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().kda_status_string(int(status)).decode()


def call(name: str, *args) -> None:
    """Call one C-ABI entry point; raise KdaError unless it returns KDA_OK."""
    st = getattr(load(), name)(*args)
    if st != KDA_OK:
        raise KdaError(st, name)


def workspace_size(name: str, *args) -> int:
    """Bytes returned by one of the *_workspace_size entry points."""
    out = ctypes.c_size_t(0)
    call(name, *args, ctypes.byref(out))
    return int(out.value)
