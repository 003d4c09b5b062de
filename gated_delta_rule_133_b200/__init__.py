"""KDA / gated-DeltaNet linear-attention layer for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in ``include/kda.h`` (``libkda.so``).  These
functions only marshal arguments (check devices, dtypes and shapes, allocate
outputs with PyTorch, pass pointers and the current CUDA stream); every step of
the computation runs in the library's CUDA kernels.  There is no CPU path.

    o, S_T = kda_chunk_fwd(q, k, v, beta, log_alpha, initial_state)
    o, S_N = kda_varlen_fwd(q, k, v, beta, log_alpha, cu_seqlens, initial_state)
    o      = kda_recurrent_step(q, k, v, beta, log_alpha, state)   # state updated in place

The output o is fp32 by default (``o_dtype=torch.bfloat16`` rounds it to bf16).
Two variants of the layer are keyword flags of the three calls (the
``KDA_MODE_*`` flags of the C ABI): ``head_gate=True`` takes one forget gate per
(token, head) -- log_alpha without its d_k axis -- and ``erase=False`` drops the
delta rule's erase term (S_t = Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T).  Two
more flags move input pre-processing into the kernels: ``normalize_qk=True``
divides every q and k row by its L2 norm, and ``gate_logits=True`` reads
log_alpha as logits z (log alpha = -softplus(z)).

The tensor-core chunk forward needs scratch memory: these calls ask the library
for its size (``kda_chunk_fwd_workspace_size`` / ``kda_varlen_fwd_workspace_size``)
and allocate it with PyTorch's caching allocator, or take a caller's uint8
``workspace`` tensor.  ``cuda_cores=True`` runs the fp32 CUDA-core kernel and
``blocks=n`` the two-stream blocked schedule (cross-checks; same results).
"""
from __future__ import annotations

import torch

from . import _lib
from ._lib import KdaError

__all__ = ["kda_chunk_fwd", "kda_chunk_fwd_noalloc", "kda_varlen_fwd", "kda_recurrent_step", "kda_check",
           "kda_chunk_bwd", "kda_varlen_bwd", "kda_dplr_fwd", "kda_dplr_varlen_fwd", "chunk_fwd_workspace_size",
           "varlen_fwd_workspace_size", "dplr_fwd_workspace_size", "KdaError"]

_DTYPES = {torch.float32: _lib.KDA_F32, torch.bfloat16: _lib.KDA_BF16}


def _ptr(t):
    return None if t is None else t.data_ptr()


def _mode(head_gate, erase, normalize_qk=False, gate_logits=False, cuda_cores=False, blocks=0):
    return ((_lib.KDA_MODE_HEAD_GATE if head_gate else 0) | (0 if erase else _lib.KDA_MODE_NO_ERASE)
            | (_lib.KDA_MODE_NORM_QK if normalize_qk else 0) | (_lib.KDA_MODE_GATE_LOGITS if gate_logits else 0)
            | (_lib.KDA_MODE_CUDA_CORES if cuda_cores else 0) | _lib.KDA_MODE_BLOCKS(int(blocks)))


def chunk_fwd_workspace_size(B, T, H, dk, dv, dtype=torch.bfloat16, chunk=64, mode=0):
    """Workspace bytes kda_chunk_fwd needs for these sizes (0 on the CUDA-core path)."""
    return _lib.workspace_size("kda_chunk_fwd_workspace_size", B, T, H, dk, dv, chunk, _DTYPES[dtype], mode)


def varlen_fwd_workspace_size(N, T, H, dk, dv, dtype=torch.bfloat16, chunk=64, mode=0):
    """Workspace bytes kda_varlen_fwd needs for N packed sequences of T tokens in all."""
    return _lib.workspace_size("kda_varlen_fwd_workspace_size", N, T, H, dk, dv, chunk, _DTYPES[dtype], mode)


def dplr_fwd_workspace_size(B, T, H, dk, dv, dtype=torch.bfloat16, chunk=64):
    """Workspace bytes kda_dplr_fwd needs for these sizes."""
    return _lib.workspace_size("kda_dplr_fwd_workspace_size", B, T, H, dk, dv, chunk, _DTYPES[dtype])


def _workspace(nbytes, workspace, device):
    """(pointer, bytes) of the scratch a call needs: the caller's uint8 tensor,
    or a fresh one from PyTorch's caching allocator."""
    if nbytes == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    if workspace.device != device or workspace.dtype != torch.uint8 or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous uint8 tensor on the inputs' device")
    return workspace.data_ptr(), workspace.numel()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check(t, name, shape, dtype, device):
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def kda_chunk_fwd(q, k, v, beta, log_alpha, initial_state=None, *, o=None, final_state=None,
                  output_final_state=True, o_dtype=torch.float32, chunk=64, stream=None,
                  head_gate=False, erase=True, normalize_qk=False, gate_logits=False,
                  workspace=None, cuda_cores=False, blocks=0):
    """Chunkwise forward over equal-length sequences.

    q, k [B, T, H, dk] and v [B, T, H, dv] (bf16 or fp32); beta [B, T, H] and
    log_alpha [B, T, H, dk] fp32 ([B, T, H] with head_gate); initial_state
    [B, H, dk, dv] fp32 or None.  Returns (o [B, T, H, dv] in o_dtype (or o's
    dtype when o is given), final_state [B, H, dk, dv] or None)."""
    return _dense_fwd("kda_chunk_fwd", q, k, v, beta, log_alpha, initial_state, o, final_state,
                      output_final_state, o_dtype, chunk, stream,
                      _mode(head_gate, erase, normalize_qk, gate_logits, cuda_cores, blocks), workspace)


def kda_chunk_fwd_noalloc(q, k, v, beta, log_alpha, initial_state=None, *, o=None, final_state=None,
                          output_final_state=True, o_dtype=torch.float32, chunk=64, stream=None):
    """kda_chunk_fwd with every intermediate in the library's fixed per-device
    area (no allocation by the library).  Calls must be ordered with respect to
    each other; raises KdaError (unsupported) when the problem does not fit."""
    return _dense_fwd("kda_chunk_fwd_noalloc", q, k, v, beta, log_alpha, initial_state, o, final_state,
                      output_final_state, o_dtype, chunk, stream)


def _dense_fwd(symbol, q, k, v, beta, log_alpha, initial_state, o, final_state, output_final_state, o_dtype,
               chunk, stream, mode=0, workspace=None):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    for t, n, s, d in ((q, "q", (B, T, H, dk), dt), (k, "k", (B, T, H, dk), dt),
                       (v, "v", (B, T, H, dv), dt), (beta, "beta", (B, T, H), torch.float32),
                       (log_alpha, "log_alpha", (B, T, H) if mode & _lib.KDA_MODE_HEAD_GATE else (B, T, H, dk),
                        torch.float32)):
        _check(t, n, s, d, dev)
    if initial_state is not None:
        _check(initial_state, "initial_state", (B, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty(B, T, H, dv, dtype=o_dtype, device=dev)
    _check(o, "o", (B, T, H, dv), o.dtype, dev)
    if o.dtype not in _DTYPES:
        raise ValueError(f"unsupported output dtype {o.dtype}")
    if final_state is None and output_final_state:
        final_state = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    if final_state is not None:
        _check(final_state, "final_state", (B, H, dk, dv), torch.float32, dev)
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(log_alpha), _ptr(initial_state), _ptr(o),
            _ptr(final_state), B, T, H, dk, dv, chunk, _DTYPES[dt], _DTYPES[o.dtype])
    if symbol == "kda_chunk_fwd_noalloc":
        _lib.call(symbol, *args, _stream(stream))
        return o, final_state
    ws = _workspace(chunk_fwd_workspace_size(B, T, H, dk, dv, dt, chunk, mode), workspace, dev)
    if mode:
        _lib.call("kda_chunk_fwd_mode", *args, mode, *ws, _stream(stream))
    else:
        _lib.call("kda_chunk_fwd", *args, *ws, _stream(stream))
    return o, final_state


def kda_varlen_fwd(q, k, v, beta, log_alpha, cu_seqlens, initial_state=None, *, o=None,
                   final_state=None, output_final_state=True, o_dtype=torch.float32, chunk=64,
                   stream=None, head_gate=False, erase=True, normalize_qk=False, gate_logits=False,
                   workspace=None, cuda_cores=False):
    """Chunkwise forward over N packed variable-length sequences.

    q, k [T, H, dk], v [T, H, dv]; beta [T, H]; log_alpha [T, H, dk] ([T, H]
    with head_gate);
    cu_seqlens [N + 1] int32 on the device; initial_state [N, H, dk, dv] or None.
    Returns (o [T, H, dv], final_state [N, H, dk, dv] or None)."""
    T, H, dk = q.shape
    dv = v.shape[-1]
    N = cu_seqlens.shape[0] - 1
    dev, dt = q.device, q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    for t, n, s, d in ((q, "q", (T, H, dk), dt), (k, "k", (T, H, dk), dt), (v, "v", (T, H, dv), dt),
                       (beta, "beta", (T, H), torch.float32),
                       (log_alpha, "log_alpha", (T, H) if head_gate else (T, H, dk), torch.float32),
                       (cu_seqlens, "cu_seqlens", (N + 1,), torch.int32)):
        _check(t, n, s, d, dev)
    if initial_state is not None:
        _check(initial_state, "initial_state", (N, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty(T, H, dv, dtype=o_dtype, device=dev)
    _check(o, "o", (T, H, dv), o.dtype, dev)
    if o.dtype not in _DTYPES:
        raise ValueError(f"unsupported output dtype {o.dtype}")
    if final_state is None and output_final_state:
        final_state = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    if final_state is not None:
        _check(final_state, "final_state", (N, H, dk, dv), torch.float32, dev)
    mode = _mode(head_gate, erase, normalize_qk, gate_logits, cuda_cores)
    ws = _workspace(varlen_fwd_workspace_size(N, T, H, dk, dv, dt, chunk, mode), workspace, dev)
    _lib.call("kda_varlen_fwd_mode" if mode else "kda_varlen_fwd", _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
              _ptr(log_alpha), _ptr(cu_seqlens), N, _ptr(initial_state), _ptr(o), _ptr(final_state), T, H, dk,
              dv, chunk, _DTYPES[dt], _DTYPES[o.dtype], *((mode,) if mode else ()), *ws, _stream(stream))
    return o, final_state


def kda_recurrent_step(q, k, v, beta, log_alpha, state, *, o=None, o_dtype=torch.float32,
                       stream=None, head_gate=False, erase=True, normalize_qk=False, gate_logits=False):
    """One decode step: q, k [N, H, dk], v [N, H, dv], beta [N, H],
    log_alpha [N, H, dk] ([N, H] with head_gate); state [N, H, dk, dv] fp32 is
    updated in place.  Returns o [N, H, dv]."""
    N, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    for t, n, s, d in ((q, "q", (N, H, dk), dt), (k, "k", (N, H, dk), dt), (v, "v", (N, H, dv), dt),
                       (beta, "beta", (N, H), torch.float32),
                       (log_alpha, "log_alpha", (N, H) if head_gate else (N, H, dk), torch.float32),
                       (state, "state", (N, H, dk, dv), torch.float32)):
        _check(t, n, s, d, dev)
    if o is None:
        o = torch.empty(N, H, dv, dtype=o_dtype, device=dev)
    _check(o, "o", (N, H, dv), o.dtype, dev)
    if o.dtype not in _DTYPES:
        raise ValueError(f"unsupported output dtype {o.dtype}")
    mode = _mode(head_gate, erase, normalize_qk, gate_logits)
    _lib.call("kda_recurrent_step_mode" if mode else "kda_recurrent_step", _ptr(q), _ptr(k), _ptr(v),
              _ptr(beta), _ptr(log_alpha), _ptr(state), _ptr(o), N, H, dk, dv, _DTYPES[dt], _DTYPES[o.dtype],
              *((mode,) if mode else ()), _stream(stream))
    return o


def _bwd_outputs(q, v, beta, nstates, H, dk, dv, want_ds0):
    dev = q.device
    f32 = dict(dtype=torch.float32, device=dev)
    grads = (torch.empty(q.shape, **f32), torch.empty(q.shape, **f32), torch.empty(v.shape, **f32),
             torch.empty(beta.shape, **f32), torch.empty(q.shape, **f32))
    ds0 = torch.empty(nstates, H, dk, dv, **f32) if want_ds0 else None
    return grads, ds0


def kda_chunk_bwd(q, k, v, beta, log_alpha, initial_state, grad_o, grad_final_state=None, *,
                  want_initial_state_grad=True, chunk=64, stream=None, workspace=None):
    """Backward of kda_chunk_fwd: gradients of sum(o * grad_o) + sum(S_T * grad_final_state).

    Inputs as for kda_chunk_fwd (plain layer); grad_o [B, T, H, dv] fp32,
    grad_final_state [B, H, dk, dv] fp32 or None.  Returns fp32
    (dq, dk, dv, dbeta, dlog_alpha, dinitial_state or None)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    for t, n, s_, d in ((q, "q", (B, T, H, dk), dt), (k, "k", (B, T, H, dk), dt), (v, "v", (B, T, H, dv), dt),
                        (beta, "beta", (B, T, H), torch.float32), (log_alpha, "log_alpha", (B, T, H, dk), torch.float32),
                        (grad_o, "grad_o", (B, T, H, dv), torch.float32)):
        _check(t, n, s_, d, dev)
    for t, n in ((initial_state, "initial_state"), (grad_final_state, "grad_final_state")):
        if t is not None:
            _check(t, n, (B, H, dk, dv), torch.float32, dev)
    (gq, gk, gv, gb, gla), gs0 = _bwd_outputs(q, v, beta, B, H, dk, dv, want_initial_state_grad)
    nbytes = _lib.workspace_size("kda_chunk_bwd_workspace_size", B, T, H, dk, dv, chunk, _DTYPES[dt])
    ws = _workspace(nbytes, workspace, dev)
    _lib.call("kda_chunk_bwd", _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(log_alpha), _ptr(initial_state),
              _ptr(grad_o), _ptr(grad_final_state), _ptr(gq), _ptr(gk), _ptr(gv), _ptr(gb), _ptr(gla), _ptr(gs0),
              B, T, H, dk, dv, chunk, _DTYPES[dt], *ws, _stream(stream))
    return gq, gk, gv, gb, gla, gs0


def kda_varlen_bwd(q, k, v, beta, log_alpha, cu_seqlens, initial_state, grad_o, grad_final_state=None, *,
                   want_initial_state_grad=True, chunk=64, stream=None, workspace=None):
    """Backward of kda_varlen_fwd (packed [T, H, ...] layouts, states [N, H, dk, dv])."""
    T, H, dk = q.shape
    dv = v.shape[-1]
    N = cu_seqlens.shape[0] - 1
    dev, dt = q.device, q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    for t, n, s_, d in ((q, "q", (T, H, dk), dt), (k, "k", (T, H, dk), dt), (v, "v", (T, H, dv), dt),
                        (beta, "beta", (T, H), torch.float32), (log_alpha, "log_alpha", (T, H, dk), torch.float32),
                        (grad_o, "grad_o", (T, H, dv), torch.float32), (cu_seqlens, "cu_seqlens", (N + 1,), torch.int32)):
        _check(t, n, s_, d, dev)
    for t, n in ((initial_state, "initial_state"), (grad_final_state, "grad_final_state")):
        if t is not None:
            _check(t, n, (N, H, dk, dv), torch.float32, dev)
    (gq, gk, gv, gb, gla), gs0 = _bwd_outputs(q, v, beta, N, H, dk, dv, want_initial_state_grad)
    nbytes = _lib.workspace_size("kda_varlen_bwd_workspace_size", N, T, H, dk, dv, chunk, _DTYPES[dt])
    ws = _workspace(nbytes, workspace, dev)
    _lib.call("kda_varlen_bwd", _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(log_alpha), _ptr(cu_seqlens), N,
              _ptr(initial_state), _ptr(grad_o), _ptr(grad_final_state), _ptr(gq), _ptr(gk), _ptr(gv), _ptr(gb),
              _ptr(gla), _ptr(gs0), T, H, dk, dv, chunk, _DTYPES[dt], *ws, _stream(stream))
    return gq, gk, gv, gb, gla, gs0


def kda_dplr_fwd(q, k, v, a, b, log_alpha, initial_state=None, *, o=None, final_state=None,
                 output_final_state=True, o_dtype=torch.float32, chunk=64, workspace=None, stream=None):
    """Diagonal-plus-low-rank transition S_t = (Diag(alpha_t) + b_t a_t^T) S_{t-1} + k_t v_t^T,
    o_t = S_t^T q_t.  q, k, a, b [B, T, H, dk], v [B, T, H, dv] (bf16 or fp32);
    log_alpha [B, T, H, dk] fp32; initial_state [B, H, dk, dv] or None.
    Returns (o, final_state or None)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    for t, n, s_, d in ((q, "q", (B, T, H, dk), dt), (k, "k", (B, T, H, dk), dt), (v, "v", (B, T, H, dv), dt),
                        (a, "a", (B, T, H, dk), dt), (b, "b", (B, T, H, dk), dt),
                        (log_alpha, "log_alpha", (B, T, H, dk), torch.float32)):
        _check(t, n, s_, d, dev)
    if initial_state is not None:
        _check(initial_state, "initial_state", (B, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty(B, T, H, dv, dtype=o_dtype, device=dev)
    _check(o, "o", (B, T, H, dv), o.dtype, dev)
    if final_state is None and output_final_state:
        final_state = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    nbytes = _lib.workspace_size("kda_dplr_fwd_workspace_size", B, T, H, dk, dv, chunk, _DTYPES[dt])
    ws = _workspace(nbytes, workspace, dev)
    _lib.call("kda_dplr_fwd", _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(log_alpha), _ptr(initial_state),
              _ptr(o), _ptr(final_state), B, T, H, dk, dv, chunk, _DTYPES[dt], _DTYPES[o.dtype], *ws,
              _stream(stream))
    return o, final_state


def kda_dplr_varlen_fwd(q, k, v, a, b, log_alpha, cu_seqlens, initial_state=None, *, o=None, final_state=None,
                        output_final_state=True, o_dtype=torch.float32, chunk=64, workspace=None, stream=None):
    """kda_dplr_fwd over N packed variable-length sequences ([T, H, ...] layouts)."""
    T, H, dk = q.shape
    dv = v.shape[-1]
    N = cu_seqlens.shape[0] - 1
    dev, dt = q.device, q.dtype
    if dt not in _DTYPES:
        raise ValueError(f"unsupported dtype {dt}")
    for t, n, s_, d in ((q, "q", (T, H, dk), dt), (k, "k", (T, H, dk), dt), (v, "v", (T, H, dv), dt),
                        (a, "a", (T, H, dk), dt), (b, "b", (T, H, dk), dt),
                        (log_alpha, "log_alpha", (T, H, dk), torch.float32), (cu_seqlens, "cu_seqlens", (N + 1,), torch.int32)):
        _check(t, n, s_, d, dev)
    if initial_state is not None:
        _check(initial_state, "initial_state", (N, H, dk, dv), torch.float32, dev)
    if o is None:
        o = torch.empty(T, H, dv, dtype=o_dtype, device=dev)
    _check(o, "o", (T, H, dv), o.dtype, dev)
    if final_state is None and output_final_state:
        final_state = torch.empty(N, H, dk, dv, dtype=torch.float32, device=dev)
    nbytes = _lib.workspace_size("kda_dplr_varlen_fwd_workspace_size", N, T, H, dk, dv, chunk, _DTYPES[dt])
    ws = _workspace(nbytes, workspace, dev)
    _lib.call("kda_dplr_varlen_fwd", _ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(b), _ptr(log_alpha), _ptr(cu_seqlens),
              N, _ptr(initial_state), _ptr(o), _ptr(final_state), T, H, dk, dv, chunk, _DTYPES[dt], _DTYPES[o.dtype],
              *ws, _stream(stream))
    return o, final_state


def kda_check(stream=None):
    """Synchronise the stream and raise if a kernel reported a device-side timeout."""
    _lib.call("kda_check", _stream(stream))
