"""Pins of the diagonal-plus-low-rank oracle (oracle/dplr.py) against routes
other than itself:

- the explicitly multiplied dense transitions Diag(alpha_t) + b_t a_t^T;
- the KDA layer, which is the special case a_t = alpha_t * k_t,
  b_t = -beta_t k_t, write key beta_t k_t (checked against oracle.recurrence,
  the C token recurrence of the layer);
- a = 0: gated linear attention's parallel form (oracle.forms.gla_closed_form
  with beta = 1);
- the chunkwise form equals the recurrence for several chunk sizes and ragged
  tails (the algebra the GPU kernel follows).
"""
import numpy as np
import pytest

import oracle
from oracle import dplr, forms


def _inputs(T, dk, dv, seed, mu=-2.0, scale_ab=0.5):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, dk)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, dk)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    a = scale_ab * rng.standard_normal((T, dk)) / np.sqrt(dk)
    b = scale_ab * rng.standard_normal((T, dk)) / np.sqrt(dk)
    la = -np.log1p(np.exp(rng.standard_normal((T, dk)) + mu))
    s0 = 0.1 * rng.standard_normal((dk, dv))
    return q, k, v, a, b, la, s0


def _err(x, y):
    return float(np.max(np.abs(x - y)) / max(np.sqrt(np.mean(y * y)), 1e-300))


def test_recurrence_equals_materialised_transitions():
    q, k, v, a, b, la, s0 = _inputs(23, 6, 5, 1)
    o, S = dplr.recurrence(q[:, None], k[:, None], v[:, None], a[:, None], b[:, None], la[:, None],
                           None, s0[None, None])
    o2, S2 = dplr.materialised(q, k, v, a, b, la, s0)
    assert _err(o[:, 0], o2) < 1e-13 and _err(S[0, 0], S2) < 1e-13


def test_kda_is_the_special_case():
    T, H, dk, dv = 40, 2, 8, 6
    rng = np.random.default_rng(2)
    q = rng.standard_normal((T, H, dk)); q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rng.standard_normal((T, H, dk)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, H))))
    la = -np.log1p(np.exp(rng.standard_normal((T, H, dk)) - 1.0))
    s0 = 0.1 * rng.standard_normal((2, H, dk, dv))
    cu = np.array([0, 17, T])
    o_kda, s_kda = oracle.recurrence(q, k, v, beta, la, cu, s0)
    a = np.exp(la) * k
    b = -beta[..., None] * k
    o, S = dplr.recurrence(q, beta[..., None] * k, v, a, b, la, cu, s0)
    assert _err(o, o_kda) < 1e-12 and _err(S, s_kda) < 1e-12
    # the transposed reading (a b^T instead of b a^T) is a different map
    o_swap, _ = dplr.recurrence(q, beta[..., None] * k, v, b, a, la, cu, s0)
    assert _err(o_swap, o_kda) > 1e-3


def test_no_low_rank_term_is_gated_linear_attention():
    q, k, v, a, b, la, s0 = _inputs(31, 7, 4, 3)
    o, _ = dplr.recurrence(q[:, None], k[:, None], v[:, None], 0 * a[:, None], b[:, None], la[:, None],
                           None, s0[None, None])
    ref = forms.gla_closed_form(q, k, v, np.ones(31), la, s0)
    assert _err(o[:, 0], ref) < 1e-12


@pytest.mark.parametrize("C", [1, 3, 16, 64])
@pytest.mark.parametrize("T", [50, 128, 131])
def test_chunkwise_equals_recurrence(C, T):
    q, k, v, a, b, la, s0 = _inputs(T, 8, 6, 10 + C + T, mu=-1.0, scale_ab=0.9)
    o, S = dplr.recurrence(q[:, None], k[:, None], v[:, None], a[:, None], b[:, None], la[:, None],
                           None, s0[None, None])
    o2, S2 = dplr.chunkwise(q, k, v, a, b, la, s0, C)
    assert _err(o2, o[:, 0]) < 1e-11 and _err(S2, S[0, 0]) < 1e-11
