"""KDA / gated-DeltaNet CPU oracle -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA product path
(``gated_delta_rule_133_b200``) never imports it, and the two share no code:
the only thing both sides see is the seeded input generator, which holds none
of the method's arithmetic.

``recurrence`` is the oracle proper: the token-by-token KDA recurrence in fp64
(``kda_oracle.c``), as stated in "Hybrid Linear Attention Architecture: Making
LLM Training and Inference More Efficient" section 3.3 and "Demystifying Hybrid
LLM Architectures" section 2.3 (read-out after the write).  ``forms`` holds
independent restatements (closed forms, brute force, the chunkwise algebra)
that pin it.  ``backward`` holds the reverse-mode gradients of the same
recurrence in fp64 (the reference for a backward pass), pinned by finite
differences of ``recurrence`` and by the closed-form gradients of causal
linear attention.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libkda_oracle.so")

_libs: dict = {}


def build(force: bool = False, mutant: int | None = None) -> str:
    """Compile the fp64 oracle with gcc (plain -O2, no fast-math, no FMA
    contraction).  ``mutant`` builds a variant with one planted mistake; only
    the oracle's own mutation tests ask for that."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    out = _LIB if mutant is None else os.path.join(_LIB_DIR, f"libkda_oracle_mutant{int(mutant)}.so")
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(_SRC)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off"]
    if mutant is not None:
        cmd.append(f"-DKDA_ORACLE_MUTANT={int(mutant)}")
    subprocess.check_call(cmd + ["-o", tmp, _SRC, "-lm", "-lpthread"])
    os.replace(tmp, out)
    return out


def _load(mutant: int | None = None):
    if mutant not in _libs:
        lib = ctypes.CDLL(build(mutant=mutant))
        dp = ctypes.POINTER(ctypes.c_double)
        lib.kda_oracle_fwd.restype = ctypes.c_int
        lib.kda_oracle_fwd.argtypes = [dp, dp, dp, dp, dp, dp,
                                       ctypes.POINTER(ctypes.c_int64),
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, dp, dp, ctypes.c_int]
        _libs[mutant] = lib
    return _libs[mutant]


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def recurrence(q, k, v, beta, log_alpha, cu_seqlens=None, initial_state=None,
               erase: bool = True, nthreads: int | None = None, _mutant: int | None = None):
    """Run the KDA recurrence in fp64.

    Token-major packed layout: q, k ``[T, H, dk]``, v ``[T, H, dv]``,
    beta ``[T, H]``, log_alpha ``[T, H, dk]``; ``cu_seqlens`` ``[N+1]``
    (default: one sequence of all T tokens); ``initial_state`` ``[N, H, dk, dv]``
    or None (zeros).  Returns ``(o [T, H, dv], final_state [N, H, dk, dv])``.
    """
    q, k, v, beta, log_alpha = map(_f64, (q, k, v, beta, log_alpha))
    T, H, dk = q.shape
    dv = v.shape[2]
    if cu_seqlens is None:
        cu_seqlens = np.array([0, T], dtype=np.int64)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    if cu[-1] != T:
        raise ValueError("cu_seqlens[-1] must equal the token count")
    s0 = None if initial_state is None else _f64(initial_state)
    if s0 is not None and s0.shape != (N, H, dk, dv):
        raise ValueError(f"initial_state shape {s0.shape} != {(N, H, dk, dv)}")
    o = np.empty((T, H, dv), dtype=np.float64)
    sT = np.empty((N, H, dk, dv), dtype=np.float64)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _load(_mutant).kda_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(log_alpha),
                                _ptr(s0), cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                N, H, dk, dv, int(bool(erase)), _ptr(o), _ptr(sT),
                                int(nthreads))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_fwd failed with code {rc}")
    return o, sT


def recurrent_step(q, k, v, beta, log_alpha, state, erase: bool = True):
    """One decode step for N independent sequences: q,k ``[N, H, dk]``,
    v ``[N, H, dv]``, beta ``[N, H]``, log_alpha ``[N, H, dk]``,
    state ``[N, H, dk, dv]``.  Returns ``(o [N, H, dv], new_state)``."""
    N = np.asarray(q).shape[0]
    cu = np.arange(N + 1, dtype=np.int64)
    return recurrence(q, k, v, beta, log_alpha, cu_seqlens=cu, initial_state=state,
                      erase=erase)
