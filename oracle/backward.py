"""Gradients of the KDA recurrence, fp64 reverse mode -- TEST INFRASTRUCTURE ONLY.

The reference for a future backward pass of the layer.  Nothing here is
imported by the CUDA path.

The forward map is the token recurrence of "Hybrid Linear Attention
Architecture: Making LLM Training and Inference More Efficient", section 3.3
(decay per channel, then erase and write), with the output read after the
write ("Demystifying Hybrid LLM Architectures", section 2.3):

    Shat_t = Diag(alpha_t) S_{t-1},   u_t = v_t - Shat_t^T k_t   (u_t = v_t with the erase off)
    S_t    = Shat_t + beta_t k_t u_t^T,   o_t = S_t^T q_t

For a scalar objective L with dL/do_t = do_t and dL/dS_T = dS_T, one step
backwards gives, with dS the gradient at S_t (after adding q_t do_t^T):

    dq_t    = S_t do_t
    dv_t    = beta_t dS^T k_t
    dbeta_t = k_t^T dS u_t
    dk_t    = beta_t dS u_t - beta_t Shat_t dS^T k_t   (the second term only with the erase)
    dShat   = dS - beta_t k_t k_t^T dS                 (likewise)
    dS_{t-1} = Diag(alpha_t) dShat,   dlog_alpha_t = alpha_t * rowsum(dShat * S_{t-1})

Shapes are those of ``oracle.recurrence``: q, k ``[T, H, dk]``, v ``[T, H, dv]``,
beta ``[T, H]``, log_alpha ``[T, H, dk]``, cu_seqlens ``[N + 1]``,
initial_state ``[N, H, dk, dv]`` (or None), do ``[T, H, dv]``, dsT
``[N, H, dk, dv]`` (or None).
"""
from __future__ import annotations

import numpy as np


def recurrence_backward(q, k, v, beta, log_alpha, cu_seqlens=None, initial_state=None, do=None, dsT=None,
                        erase: bool = True):
    """Returns (dq, dk, dv, dbeta, dlog_alpha, ds0) of L = sum(o * do) + sum(S_T * dsT)."""
    q, k, v, beta, log_alpha = (np.asarray(a, dtype=np.float64) for a in (q, k, v, beta, log_alpha))
    T, H, dk = q.shape
    dv_ = v.shape[2]
    cu = np.array([0, T]) if cu_seqlens is None else np.asarray(cu_seqlens, dtype=np.int64)
    N = len(cu) - 1
    do = np.zeros((T, H, dv_)) if do is None else np.asarray(do, dtype=np.float64)
    grads = [np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros_like(beta), np.zeros_like(log_alpha)]
    dq, dkk, dvv, dbeta, dla = grads
    ds0 = np.zeros((N, H, dk, dv_))
    alpha = np.exp(log_alpha)
    for n in range(N):
        a, b = int(cu[n]), int(cu[n + 1])
        for h in range(H):
            S = np.zeros((dk, dv_)) if initial_state is None else np.array(initial_state[n, h], dtype=np.float64)
            prev = []                                  # S_{t-1} of every token
            for t in range(a, b):
                prev.append(S)
                Shat = alpha[t, h][:, None] * S
                u = v[t, h] - (Shat.T @ k[t, h] if erase else 0.0)
                S = Shat + beta[t, h] * np.outer(k[t, h], u)
            dS = np.zeros((dk, dv_)) if dsT is None else np.array(dsT[n, h], dtype=np.float64)
            for t in range(b - 1, a - 1, -1):
                Sp = prev[t - a]
                Shat = alpha[t, h][:, None] * Sp
                u = v[t, h] - (Shat.T @ k[t, h] if erase else 0.0)
                St = Shat + beta[t, h] * np.outer(k[t, h], u)
                dq[t, h] = St @ do[t, h]
                dS = dS + np.outer(q[t, h], do[t, h])
                dSk = dS.T @ k[t, h]                   # [dv]
                dvv[t, h] = beta[t, h] * dSk
                dbeta[t, h] = k[t, h] @ dS @ u
                dkk[t, h] = beta[t, h] * (dS @ u)
                dShat = dS
                if erase:
                    dkk[t, h] -= beta[t, h] * (Shat @ dSk)
                    dShat = dS - beta[t, h] * np.outer(k[t, h], dSk)
                dla[t, h] = alpha[t, h] * np.sum(dShat * Sp, axis=1)
                dS = alpha[t, h][:, None] * dShat
            ds0[n, h] = dS
    return dq, dkk, dvv, dbeta, dla, ds0
