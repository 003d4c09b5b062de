"""Diagonal-plus-low-rank transition -- TEST INFRASTRUCTURE ONLY.

The "finer granularity" gate of "Hybrid Linear Attention Architecture: Making
LLM Training and Inference More Efficient", section 3.3 (also "Hybrid Linear
Attention Architecture: Technical Deep Dive ...", the RWKV-7 line of its
comparison, and "Linear Attention Architecture Deep Dive", section 3.4): a
low-rank correction on top of the element-wise decay,

    pages' orientation (S is d_v x d_k):   S_t = S_{t-1} (Diag(alpha_t) + a_t b_t^T) + v_t k_t^T

and, transposed to this library's d_k x d_v state,

    S_t = (Diag(alpha_t) + b_t a_t^T) S_{t-1} + k_t v_t^T,      o_t = S_t^T q_t

(read-out after the write, as for the layer).  Nothing here is imported by the
CUDA path.  All arithmetic is fp64 NumPy.

Shapes for one sequence and one head: q, k, a, b, log_alpha [T, dk],
v [T, dv], s0 [dk, dv].  ``recurrence`` takes the packed multi-head layout of
``oracle.recurrence``: [T, H, d] with ``cu_seqlens``.
"""
from __future__ import annotations

import numpy as np


def recurrence(q, k, v, a, b, log_alpha, cu_seqlens=None, initial_state=None):
    """Token-by-token fp64 recurrence; returns (o [T, H, dv], S_N [N, H, dk, dv])."""
    q, k, v, a, b, log_alpha = (np.asarray(x, dtype=np.float64) for x in (q, k, v, a, b, log_alpha))
    T, H, dk = q.shape
    dv = v.shape[2]
    cu = np.array([0, T]) if cu_seqlens is None else np.asarray(cu_seqlens, dtype=np.int64)
    N = len(cu) - 1
    o = np.zeros((T, H, dv))
    sN = np.zeros((N, H, dk, dv))
    alpha = np.exp(log_alpha)
    for n in range(N):
        for h in range(H):
            S = np.zeros((dk, dv)) if initial_state is None else np.array(initial_state[n, h], dtype=np.float64)
            for t in range(int(cu[n]), int(cu[n + 1])):
                # (Diag(alpha) + b a^T) S + k v^T, the low-rank part as b (a^T S)
                S = alpha[t, h][:, None] * S + np.outer(b[t, h], a[t, h] @ S) + np.outer(k[t, h], v[t, h])
                o[t, h] = S.T @ q[t, h]
            sN[n, h] = S
    return o, sN


def materialised(q, k, v, a, b, log_alpha, s0):
    """One (sequence, head): S_t = M_t S_{t-1} + k_t v_t^T with the dense
    transitions M_t = Diag(alpha_t) + b_t a_t^T multiplied out explicitly."""
    T, dk = q.shape
    S = np.array(s0, dtype=np.float64)
    o = np.zeros((T, v.shape[1]))
    for t in range(T):
        M = np.diag(np.exp(log_alpha[t])) + np.outer(b[t], a[t])
        S = M @ S + np.outer(k[t], v[t])
        o[t] = S.T @ q[t]
    return o, S


def chunkwise(q, k, v, a, b, log_alpha, s0, C):
    """The chunkwise-parallel form, fp64, one (sequence, head).

    Inside a chunk, with G the inclusive cumulative sum of log alpha, Gx its
    exclusive one (the decay before token s), u_s = S_{s-1}^T a_s and
    S_r = e^{G_r} S_0 + sum_{s<=r} e^{G_r - G_s} (b_s u_s^T + k_s v_s^T):

      u_s = (e^{Gx_s} a_s)^T S_0 + sum_{t<s} [a_s . (e^{Gx_s - G_t} b_t)] u_t
                                 + sum_{t<s} [a_s . (e^{Gx_s - G_t} k_t)] v_t
      => U = T (Ah S_0 + A_ak V),  T = (I - A_ab)^-1   (unit lower triangular)
      O     = (e^G q) S_0 + P_qb U + P_qk V          (P_* include the diagonal)
      S_end = e^{G_last} S_0 + (e^{G_last - G} b)^T U + (e^{G_last - G} k)^T V
    Returns (o [T, dv], S_T)."""
    T = q.shape[0]
    S = np.array(s0, dtype=np.float64)
    o = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        c1 = min(T, c0 + C)
        Q, K, V, Aa, Bb = q[c0:c1], k[c0:c1], v[c0:c1], a[c0:c1], b[c0:c1]
        G = np.cumsum(log_alpha[c0:c1], axis=0)
        Gx = G - log_alpha[c0:c1]
        L = c1 - c0
        strict = np.arange(L)[:, None] > np.arange(L)[None, :]
        low = np.arange(L)[:, None] >= np.arange(L)[None, :]
        Dx = np.exp(Gx[:, None, :] - G[None, :, :])          # [s, t, c]: decay from after t to before s
        D = np.exp(G[:, None, :] - G[None, :, :])            # [r, s, c]: decay from after s through r
        A_ab = np.einsum("sc,tc,stc->st", Aa, Bb, np.where(strict[:, :, None], Dx, 0.0))
        A_ak = np.einsum("sc,tc,stc->st", Aa, K, np.where(strict[:, :, None], Dx, 0.0))
        P_qb = np.einsum("rc,sc,rsc->rs", Q, Bb, np.where(low[:, :, None], D, 0.0))
        P_qk = np.einsum("rc,sc,rsc->rs", Q, K, np.where(low[:, :, None], D, 0.0))
        Tm = np.linalg.inv(np.eye(L) - A_ab)
        U = Tm @ ((np.exp(Gx) * Aa) @ S + A_ak @ V)
        o[c0:c1] = (np.exp(G) * Q) @ S + P_qb @ U + P_qk @ V
        F = np.exp(G[-1][None, :] - G)
        S = np.exp(G[-1])[:, None] * S + (F * Bb).T @ U + (F * K).T @ V
    return o, S
