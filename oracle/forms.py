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


def chunkwise_backward(q, k, v, beta, log_alpha, s0, do, dsT, C):
    """Gradients of L = sum(o * do) + sum(S_T * dsT) through the chunkwise
    algorithm of ``chunkwise`` (fp64, one (sequence, head)): the adjoint of
    each chunk's map, a reverse scan over chunks carrying dS.  Per chunk, with
    E = exp(G), gamma = exp(G_last), Qh = E * Q, Kh = E * K, Kn = K / E,
    Kl = gamma * Kn, A = beta strictly-lower(Kh Kn^T), P = lower-incl(Qh Kn^T),
    T = (I + A)^-1, Y = beta (V - Kh S), U = T Y:
      O = Qh S + P U,   S_next = Diag(gamma) S + Kl^T U.
    Returns (dq, dk, dv, dbeta, dlog_alpha, ds0); the same quantities as
    ``oracle.backward.recurrence_backward`` by a different route."""
    T = q.shape[0]
    dk_, dv_ = q.shape[1], v.shape[1]
    starts = list(range(0, T, C))
    S = np.array(s0, dtype=np.float64)
    states = []
    for c0 in starts:                                   # forward: the state entering each chunk
        states.append(S)
        c1 = min(T, c0 + C)
        G = np.cumsum(log_alpha[c0:c1], axis=0)
        E, gam = np.exp(G), np.exp(G[-1])
        L = c1 - c0
        Kh, Kn = k[c0:c1] * E, k[c0:c1] / E
        A = beta[c0:c1, None] * np.tril(Kh @ Kn.T, -1)
        U = np.linalg.inv(np.eye(L) + A) @ (beta[c0:c1, None] * (v[c0:c1] - Kh @ S))
        S = gam[:, None] * S + (gam[None, :] * Kn).T @ U
    grads = [np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros_like(beta), np.zeros_like(log_alpha)]
    gq, gk, gv, gb, gg = grads
    dS = np.zeros((dk_, dv_)) if dsT is None else np.array(dsT, dtype=np.float64)
    for ci in range(len(starts) - 1, -1, -1):
        c0 = starts[ci]
        c1 = min(T, c0 + C)
        L = c1 - c0
        S = states[ci]
        Q, K, V, b, dO = q[c0:c1], k[c0:c1], v[c0:c1], beta[c0:c1], do[c0:c1]
        G = np.cumsum(log_alpha[c0:c1], axis=0)
        E, En, gam = np.exp(G), np.exp(-G), np.exp(G[-1])
        Qh, Kh, Kn = Q * E, K * E, K * En
        Kl = Kn * gam[None, :]
        low, strict = np.tril(np.ones((L, L))), np.tril(np.ones((L, L)), -1)
        MA, MP = Kh @ Kn.T, Qh @ Kn.T
        A, P = b[:, None] * MA * strict, MP * low
        Tm = np.linalg.inv(np.eye(L) + A)
        X = Kh @ S
        Y = b[:, None] * (V - X)
        U = Tm @ Y
        dSn = dS
        # adjoint of O = Qh S + P U and S_next = Diag(gamma) S + Kl^T U
        dU = P.T @ dO + Kl @ dSn
        dP = (dO @ U.T) * low
        dKl = U @ dSn.T
        dgam = np.sum(dSn * S, axis=1)
        dS = gam[:, None] * dSn + Qh.T @ dO
        dQh = dO @ S.T
        # U = T Y,  Y = beta (V - Kh S)
        dY = Tm.T @ dU
        dTm = dU @ Y.T
        gv[c0:c1] = b[:, None] * dY
        dX = -b[:, None] * dY
        db = np.sum((V - X) * dY, axis=1)
        dKh = dX @ S.T
        dS = dS + Kh.T @ dX
        # T = (I + A)^-1,  A = beta strictly-lower(Kh Kn^T),  P = lower-incl(Qh Kn^T)
        dA = -(Tm.T @ dTm @ Tm.T) * strict
        db += np.sum(MA * strict * dA, axis=1)
        dMA = b[:, None] * dA
        dKh += dMA @ Kn
        dKn = dMA.T @ Kh + dP.T @ Qh + dKl * gam[None, :]
        dQh += dP @ Kn
        dgam += np.sum(dKl * Kn, axis=0)
        # Qh = E Q, Kh = E K, Kn = K / E, gamma = E[-1]; G = cumsum(log alpha)
        gq[c0:c1] = dQh * E
        gk[c0:c1] = dKh * E + dKn * En
        dG = dQh * Qh + dKh * Kh - dKn * Kn
        dG[-1] += dgam * gam
        gg[c0:c1] = np.cumsum(dG[::-1], axis=0)[::-1]
        gb[c0:c1] = db
    return gq, gk, gv, gb, gg, dS
