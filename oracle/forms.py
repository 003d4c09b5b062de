"""Independent restatements of the KDA layer -- TEST INFRASTRUCTURE ONLY.

Each function computes, by a route other than the token recurrence in
``kda_oracle.c``, a quantity the recurrence must reproduce.  They pin the
oracle (and nothing here is imported by the CUDA path).  All arithmetic is
fp64 NumPy, one (sequence, head) at a time, on small inputs.

Shapes for one sequence and one head: q, k ``[T, dk]``, v ``[T, dv]``,
beta ``[T]``, log_alpha ``[T, dk]``, s0 ``[dk, dv]``.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np


def linear_attention_closed_form(q, k, v, beta, s0):
    """Accumulate-only linear attention ("Hybrid Linear Attention Architecture:
    Making LLM Training and Inference More Efficient", section 3.1), written as
    causal masked attention without softmax:
    o_t = S0^T q_t + sum_{s<=t} beta_s v_s (k_s . q_t).
    This is the KDA recurrence with alpha = 1 and the erase term dropped."""
    scores = (q @ k.T) * beta[None, :]
    mask = np.tril(np.ones((q.shape[0], q.shape[0])))
    return q @ s0 + (scores * mask) @ v


def gla_closed_form(q, k, v, beta, log_alpha, s0):
    """Per-channel decay, no erase (the element-wise-gated form on the same
    page, section 3.3, transposed to a d_k x d_v state).  Parallel form:
    o_t = (exp(G_t) * q_t)^T S0 + sum_{s<=t} beta_s v_s sum_c q_tc k_sc exp(G_tc - G_sc),
    with G_t the inclusive cumulative sum of log alpha."""
    T = q.shape[0]
    G = np.cumsum(log_alpha, axis=0)
    o = (q * np.exp(G)) @ s0
    for t in range(T):
        for s in range(t + 1):
            w = np.sum(q[t] * k[s] * np.exp(G[t] - G[s]))
            o[t] += beta[s] * w * v[s]
    return o


def deltanet_loop_dv_dk(q, k, v, beta, s0):
    """The delta-rule inference loop of "Demystifying Hybrid LLM Architectures",
    section 2.3, kept in that page's orientation: a (d_v, d_k) memory,
    retrieve S @ k, write beta * outer(v - retrieved, k), then read S @ q.
    Returns (o [T, dv], final state transposed back to [dk, dv])."""
    S = np.array(s0, dtype=np.float64).T.copy()          # (dv, dk)
    out = np.zeros((q.shape[0], S.shape[0]))
    for t in range(q.shape[0]):
        retrieved = S @ k[t]
        S = S + beta[t] * np.outer(v[t] - retrieved, k[t])
        out[t] = S @ q[t]
    return out, S.T


def transition(k_t, beta_t, alpha_t):
    """Dense KDA transition M_t = (I - beta_t k_t k_t^T) Diag(alpha_t)
    ("... Making LLM Training and Inference More Efficient", section 3.3)."""
    dk = k_t.shape[0]
    return (np.eye(dk) - beta_t * np.outer(k_t, k_t)) @ np.diag(alpha_t)


def materialised_product(q, k, v, beta, log_alpha, s0):
    """Unrolled solution of S_t = M_t S_{t-1} + beta_t k_t v_t^T:
    S_t = Phi(t,0) S0 + sum_{s<=t} Phi(t,s) beta_s k_s v_s^T with
    Phi(t,s) = M_t ... M_{s+1} formed as explicit dense matrix products.
    Returns (o [T, dv], S_T)."""
    T, dk = k.shape
    alpha = np.exp(log_alpha)
    M = [transition(k[t], beta[t], alpha[t]) for t in range(T)]
    o = np.zeros((T, v.shape[1]))
    S_t = None
    for t in range(T):
        phi = np.eye(dk)                     # Phi(t, t)
        acc = beta[t] * np.outer(k[t], v[t])
        for s in range(t - 1, -1, -1):       # build Phi(t, s) = Phi(t, s+1) M_{s+1}
            phi = phi @ M[s + 1]
            acc = acc + phi @ (beta[s] * np.outer(k[s], v[s]))
        phi = phi @ M[0]                     # Phi(t, -1): acts on S0
        S_t = phi @ s0 + acc
        o[t] = S_t.T @ q[t]
    return o, (s0.copy() if S_t is None else S_t)


def exact_recurrence_fraction(q, k, v, beta, alpha, s0):
    """Exact rational brute force of the KDA update for tiny cases, using
    Python Fractions and dense matrices (no floating point at all).
    alpha is given directly (not its logarithm).  Returns lists of Fractions."""
    dk, dv = len(s0), len(s0[0])
    S = [[Fraction(x) for x in row] for row in s0]
    outs = []
    for t in range(len(q)):
        M = [[(Fraction(int(i == j)) - Fraction(beta[t]) * Fraction(k[t][i]) * Fraction(k[t][j]))
              * Fraction(alpha[t][j]) for j in range(dk)] for i in range(dk)]
        S = [[sum(M[i][m] * S[m][j] for m in range(dk))
              + Fraction(beta[t]) * Fraction(k[t][i]) * Fraction(v[t][j])
              for j in range(dv)] for i in range(dk)]
        outs.append([sum(S[i][j] * Fraction(q[t][i]) for i in range(dk)) for j in range(dv)])
    return outs, S


def chunkwise(q, k, v, beta, log_alpha, s0, C):
    """The chunkwise-parallel algorithm, fp64, one (sequence, head).

    Reading of the chunk recurrence printed (garbled) in "Hybrid Linear
    Attention Architecture: Making LLM Training and Inference More Efficient",
    section IV, "... Technical Deep Dive ...", section 4, and "Linear Attention
    Architecture Deep Dive", section 5.  Per chunk, with G the inclusive
    cumulative sum of log alpha inside the chunk:
      A[r,s]  = beta_r sum_c k_rc k_sc exp(G_rc - G_sc)   (s < r, else 0)
      T       = (I + A)^-1                                 (UT transform)
      W       = T diag(beta) (exp(G) * K),  U = T diag(beta) V
      V'      = U - W S                                    ("residual correction")
      O       = (exp(G) * Q) S + Tril_incl(P) V',  P[r,s] = sum_c q_rc k_sc exp(G_rc - G_sc)
      S_next  = Diag(exp(G_last)) S + (exp(G_last - G) * K)^T V'
    The last chunk may be shorter than C.  Returns (o [T, dv], S_T)."""
    T = q.shape[0]
    S = np.array(s0, dtype=np.float64)
    o = np.zeros((T, v.shape[1]))
    for c0 in range(0, T, C):
        c1 = min(T, c0 + C)
        Q, K, V = q[c0:c1], k[c0:c1], v[c0:c1]
        b = beta[c0:c1]
        G = np.cumsum(log_alpha[c0:c1], axis=0)
        L = c1 - c0
        D = np.exp(G[:, None, :] - G[None, :, :])          # [r, s, c] relative decay
        KK = np.einsum("rc,sc,rsc->rs", K, K, np.where(np.arange(L)[:, None, None] > np.arange(L)[None, :, None], D, 0.0))
        A = b[:, None] * KK
        P = np.einsum("rc,sc,rsc->rs", Q, K, np.where(np.arange(L)[:, None, None] >= np.arange(L)[None, :, None], D, 0.0))
        Tm = np.linalg.inv(np.eye(L) + A)
        W = Tm @ (b[:, None] * (np.exp(G) * K))
        U = Tm @ (b[:, None] * V)
        Vp = U - W @ S
        o[c0:c1] = (np.exp(G) * Q) @ S + P @ Vp
        S = np.exp(G[-1])[:, None] * S + (np.exp(G[-1][None, :] - G) * K).T @ Vp
    return o, S
