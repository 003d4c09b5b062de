"""Pins of the fp64 reverse-mode gradients of the recurrence (oracle/backward.py).

- Central finite differences of L = sum(o * do) + sum(S_T * dsT), evaluated
  with the forward oracle (the C recurrence, a separate code path), for every
  input element of a tiny two-sequence problem, with and without the erase
  term.
- Causal linear attention (alpha = 1, no erase) has closed-form gradients of
  the scores-times-values form of "Hybrid Linear Attention Architecture: ...",
  section 3.1.
- The adjoint of the chunkwise algorithm (``oracle.forms.chunkwise_backward``:
  a reverse scan over chunks carrying dS plus per-chunk local gradients, the
  blueprint of a backward pass) equals the token-level gradients for chunk
  sizes 1, 3, 4 and 16 with a ragged last chunk.
"""
import numpy as np
import pytest

import oracle
from oracle.backward import recurrence_backward


def _problem(seed, T=6, H=2, dk=3, dv=2):
    rng = np.random.default_rng(seed)
    cu = np.array([0, 2, T])
    x = {
        "q": rng.standard_normal((T, H, dk)),
        "k": rng.standard_normal((T, H, dk)) * 0.7,
        "v": rng.standard_normal((T, H, dv)),
        "beta": rng.uniform(0.1, 0.9, (T, H)),
        "log_alpha": -rng.uniform(0.05, 1.0, (T, H, dk)),
        "s0": rng.standard_normal((2, H, dk, dv)) * 0.5,
    }
    do = rng.standard_normal((T, H, dv))
    dsT = rng.standard_normal((2, H, dk, dv))
    return x, cu, do, dsT


def _loss(x, cu, do, dsT, erase):
    o, sT = oracle.recurrence(x["q"], x["k"], x["v"], x["beta"], x["log_alpha"], cu, x["s0"], erase=erase)
    return float(np.sum(o * do) + np.sum(sT * dsT))


@pytest.mark.parametrize("erase", [True, False])
def test_gradients_match_finite_differences(erase):
    x, cu, do, dsT = _problem(3)
    got = dict(zip(("q", "k", "v", "beta", "log_alpha", "s0"),
                   recurrence_backward(x["q"], x["k"], x["v"], x["beta"], x["log_alpha"], cu, x["s0"], do, dsT,
                                       erase=erase)))
    h = 1e-6
    for name, arr in x.items():
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            keep = arr[idx]
            arr[idx] = keep + h
            lp = _loss(x, cu, do, dsT, erase)
            arr[idx] = keep - h
            lm = _loss(x, cu, do, dsT, erase)
            arr[idx] = keep
            fd[idx] = (lp - lm) / (2 * h)
        scale = max(1.0, float(np.abs(fd).max()))
        assert np.abs(got[name] - fd).max() <= 1e-6 * scale, name


def test_linear_attention_closed_form_gradients():
    """alpha = 1, no erase: o_t = S0^T q_t + sum_{s<=t} beta_s v_s (k_s . q_t)."""
    rng = np.random.default_rng(5)
    T, dk, dv = 7, 4, 3
    q, k, v = rng.standard_normal((T, dk)), rng.standard_normal((T, dk)), rng.standard_normal((T, dv))
    beta = rng.uniform(0.1, 1.0, T)
    s0 = rng.standard_normal((dk, dv))
    do = rng.standard_normal((T, dv))
    mask = np.tril(np.ones((T, T)))                       # [t, s]: s <= t
    qk = (q @ k.T) * mask                                 # k_s . q_t
    vdo = (do @ v.T) * mask                               # v_s . do_t
    want = {
        "q": do @ s0.T + (vdo * beta[None, :]) @ k,
        "k": beta[:, None] * (vdo.T @ q),
        "v": beta[:, None] * (qk.T @ do),
        "beta": np.sum(qk * vdo, axis=0),
        "s0": q.T @ do,
    }
    got = recurrence_backward(q[:, None], k[:, None], v[:, None], beta[:, None], np.zeros((T, 1, dk)), None,
                              s0[None, None], do[:, None], None, erase=False)
    got = dict(zip(("q", "k", "v", "beta", "log_alpha", "s0"), got))
    for name in ("q", "k", "v", "beta"):
        assert np.allclose(got[name][:, 0], want[name], rtol=1e-12, atol=1e-12), name
    assert np.allclose(got["s0"][0, 0], want["s0"], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("C", [1, 3, 4, 16])
def test_chunkwise_backward_matches_token_backward(C):
    """The chunk algebra's adjoint (a reverse scan over chunks plus per-chunk
    local gradients) gives the token recurrence's gradients, ragged last chunk
    included."""
    from oracle.forms import chunkwise_backward
    rng = np.random.default_rng(7 + C)
    T, dk, dv = 11, 4, 3
    q, k, v = rng.standard_normal((T, dk)), rng.standard_normal((T, dk)) * 0.6, rng.standard_normal((T, dv))
    beta = rng.uniform(0.1, 0.9, T)
    la = -rng.uniform(0.02, 0.3, (T, dk))
    s0 = rng.standard_normal((dk, dv))
    do, dsT = rng.standard_normal((T, dv)), rng.standard_normal((dk, dv))
    want = recurrence_backward(q[:, None], k[:, None], v[:, None], beta[:, None], la[:, None], None,
                               s0[None, None], do[:, None], dsT[None, None])
    got = chunkwise_backward(q, k, v, beta, la, s0, do, dsT, C)
    for name, w, g in zip(("q", "k", "v", "beta", "log_alpha"), want[:5], got[:5]):
        assert np.allclose(g, w[:, 0], rtol=1e-10, atol=1e-10), name
    assert np.allclose(got[5], want[5][0, 0], rtol=1e-10, atol=1e-10)
