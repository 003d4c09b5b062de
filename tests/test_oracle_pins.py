"""Pins for the fp64 oracle (CPU only).

The oracle is the token recurrence of the KDA layer.  Each test below checks it
against something other than itself: a textbook special case, a closed form, an
exact rational brute force, an explicitly materialised product of transition
matrices, the other orientation of the pages' own delta-rule loop, or the
chunkwise algebra.  ``test_mutants_are_caught`` plants plausible mistakes in
the oracle and shows each one fails at least one of these pins.
"""
import numpy as np
import pytest

import oracle
from oracle import forms


def _rand_case(rng, T, dk, dv, gate_mu=-1.0, s0_std=0.3, normalise=True):
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    if normalise:
        q /= np.linalg.norm(q, axis=1, keepdims=True)
        k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(T)))
    log_alpha = -np.logaddexp(0.0, rng.standard_normal((T, dk)) + gate_mu)
    s0 = rng.standard_normal((dk, dv)) * s0_std
    return q, k, v, beta, log_alpha, s0


def _run(q, k, v, beta, log_alpha, s0, erase=True, mutant=None):
    """Oracle on one (sequence, head)."""
    o, sT = oracle.recurrence(q[:, None], k[:, None], v[:, None], beta[:, None],
                              log_alpha[:, None], initial_state=s0[None, None],
                              erase=erase, _mutant=mutant)
    return o[:, 0], sT[0, 0]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_vanilla_linear_attention(seed):
    """alpha = 1 and erase off: causal linear attention, closed form."""
    rng = np.random.default_rng(seed)
    q, k, v, beta, _, s0 = _rand_case(rng, 17, 6, 5)
    o, sT = _run(q, k, v, beta, np.zeros_like(q), s0, erase=False)
    np.testing.assert_allclose(o, forms.linear_attention_closed_form(q, k, v, beta, s0),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sT, s0 + (beta[:, None] * k).T @ v, rtol=1e-12, atol=1e-12)
    # beta = 1 is the accumulate-only rule S_t = S_{t-1} + k_t v_t^T
    o1, _ = _run(q, k, v, np.ones_like(beta), np.zeros_like(q), s0, erase=False)
    np.testing.assert_allclose(o1, q @ s0 + np.tril(q @ k.T) @ v, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_gated_linear_attention(seed):
    """Per-channel decay with erase off: the parallel (masked, decayed) form."""
    rng = np.random.default_rng(seed)
    q, k, v, beta, log_alpha, s0 = _rand_case(rng, 13, 5, 4)
    o, _ = _run(q, k, v, beta, log_alpha, s0, erase=False)
    np.testing.assert_allclose(o, forms.gla_closed_form(q, k, v, beta, log_alpha, s0),
                               rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_deltanet(seed):
    """alpha = 1: the delta rule, against the pages' (d_v, d_k) inference loop."""
    rng = np.random.default_rng(seed)
    q, k, v, beta, _, s0 = _rand_case(rng, 21, 7, 4, normalise=(seed != 2))
    o, sT = _run(q, k, v, beta, np.zeros_like(q), s0)
    o_ref, s_ref = forms.deltanet_loop_dv_dk(q, k, v, beta, s0)
    np.testing.assert_allclose(o, o_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(sT, s_ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("seed,T,dk,dv", [(0, 9, 5, 3), (1, 12, 4, 6), (2, 7, 8, 8)])
def test_materialised_transition_product(seed, T, dk, dv):
    """Full KDA: S_T and every o_t equal the unrolled product of the dense
    transitions M_t = (I - beta_t k_t k_t^T) Diag(alpha_t)."""
    rng = np.random.default_rng(seed)
    q, k, v, beta, log_alpha, s0 = _rand_case(rng, T, dk, dv)
    o, sT = _run(q, k, v, beta, log_alpha, s0)
    o_ref, s_ref = forms.materialised_product(q, k, v, beta, log_alpha, s0)
    np.testing.assert_allclose(o, o_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(sT, s_ref, rtol=1e-11, atol=1e-12)


def test_decay_then_erase_order():
    """The pages apply the per-channel decay before the erase; the other order
    (Diag(alpha)(I - beta k k^T)) gives a clearly different state."""
    rng = np.random.default_rng(7)
    q, k, v, beta, log_alpha, s0 = _rand_case(rng, 6, 4, 3, gate_mu=0.0)
    _, sT = _run(q, k, v, beta, log_alpha, s0)
    S = s0.copy()
    for t in range(6):
        a = np.exp(log_alpha[t])
        S = np.diag(a) @ (np.eye(4) - beta[t] * np.outer(k[t], k[t])) @ S + beta[t] * np.outer(k[t], v[t])
    assert np.max(np.abs(S - sT)) > 1e-3


def test_exact_rational_example():
    """d_k = d_v = 2, three tokens, rational inputs: exact Fraction brute force."""
    q = [[1, 0], [0.5, 0.5], [0, 1]]
    k = [[0.6, 0.8], [1, 0], [0.8, -0.6]]
    v = [[1, 2], [-1, 0.5], [0.25, -2]]
    beta = [0.5, 0.75, 1.0]
    alpha = [[1.0, 0.5], [0.25, 1.0], [0.5, 0.5]]
    s0 = [[0.5, -1.0], [2.0, 0.25]]
    outs, S = forms.exact_recurrence_fraction(q, k, v, beta, alpha, s0)
    arr = np.array
    o, sT = _run(arr(q, float), arr(k, float), arr(v, float), arr(beta, float),
                 np.log(arr(alpha, float)), arr(s0, float))
    np.testing.assert_allclose(o, np.array([[float(x) for x in r] for r in outs]), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(sT, np.array([[float(x) for x in r] for r in S]), rtol=1e-14, atol=1e-15)


def test_zero_beta_unit_alpha_is_identity():
    rng = np.random.default_rng(3)
    q, k, v, _, _, s0 = _rand_case(rng, 11, 6, 5)
    o, sT = _run(q, k, v, np.zeros(11), np.zeros_like(q), s0)
    assert np.array_equal(sT, s0)
    np.testing.assert_allclose(o, q @ s0, rtol=1e-14, atol=1e-15)


def test_full_write_is_exact():
    """beta = 1 and a unit key: after the token, the key retrieves exactly v."""
    rng = np.random.default_rng(4)
    q, k, v, _, log_alpha, s0 = _rand_case(rng, 8, 6, 5)
    S = s0
    for t in range(8):
        _, S = _run(q[t:t + 1], k[t:t + 1], v[t:t + 1], np.ones(1), log_alpha[t:t + 1], S)
        np.testing.assert_allclose(S.T @ k[t], v[t], rtol=1e-12, atol=1e-12)


def test_linearity_in_state_and_values():
    rng = np.random.default_rng(5)
    q, k, v, beta, log_alpha, s0 = _rand_case(rng, 15, 6, 4)
    o1, s1 = _run(q, k, v, beta, log_alpha, s0)
    o2, s2 = _run(q, k, -2.5 * v, beta, log_alpha, -2.5 * s0)
    np.testing.assert_allclose(o2, -2.5 * o1, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s2, -2.5 * s1, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("C", [1, 4, 16, 64])
def test_chunkwise_algebra_equals_recurrence(C):
    """The chunkwise form (the reading of the pages' garbled chunk formula that
    the CUDA kernels implement) reproduces the recurrence, including a ragged
    last chunk and the strong-forgetting gate distribution."""
    rng = np.random.default_rng(C)
    for T, mu in ((100, -3.0), (130, -1.0)):
        q, k, v, beta, log_alpha, s0 = _rand_case(rng, T, 16, 12, gate_mu=mu)
        o, sT = _run(q, k, v, beta, log_alpha, s0)
        o_c, s_c = forms.chunkwise(q, k, v, beta, log_alpha, s0, C)
        np.testing.assert_allclose(o_c, o, rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(s_c, sT, rtol=1e-9, atol=1e-11)


def test_varlen_and_split_resume():
    """Packed sequences equal separate runs; a split run resumed from the
    carried state equals one pass."""
    rng = np.random.default_rng(6)
    H, dk, dv = 3, 8, 6
    lens = [5, 1, 17, 0, 9]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T = cu[-1]
    q = rng.standard_normal((T, H, dk)); k = rng.standard_normal((T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    beta = rng.uniform(0, 1, (T, H))
    log_alpha = -rng.uniform(0, 0.5, (T, H, dk))
    s0 = rng.standard_normal((len(lens), H, dk, dv))
    o, sT = oracle.recurrence(q, k, v, beta, log_alpha, cu, s0)
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        on, sn = oracle.recurrence(q[a:b], k[a:b], v[a:b], beta[a:b], log_alpha[a:b],
                                   None, s0[n:n + 1])
        assert np.array_equal(on, o[a:b]) and np.array_equal(sn[0], sT[n])
    # split-resume on sequence 2
    a, b, m = cu[2], cu[3], cu[2] + 7
    o1, s1 = oracle.recurrence(q[a:m], k[a:m], v[a:m], beta[a:m], log_alpha[a:m], None, s0[2:3])
    o2, s2 = oracle.recurrence(q[m:b], k[m:b], v[m:b], beta[m:b], log_alpha[m:b], None, s1)
    assert np.array_equal(np.concatenate([o1, o2]), o[a:b]) and np.array_equal(s2[0], sT[2])
    # an empty sequence returns its initial state untouched
    assert np.array_equal(sT[3], s0[3])


def test_recurrent_step_is_one_token():
    rng = np.random.default_rng(8)
    N, H, dk, dv = 4, 2, 6, 5
    q = rng.standard_normal((N, H, dk)); k = rng.standard_normal((N, H, dk))
    v = rng.standard_normal((N, H, dv)); beta = rng.uniform(0, 1, (N, H))
    la = -rng.uniform(0, 1, (N, H, dk)); S = rng.standard_normal((N, H, dk, dv))
    o, S1 = oracle.recurrent_step(q, k, v, beta, la, S)
    for n in range(N):
        for h in range(H):
            o_ref, s_ref = forms.materialised_product(q[n, h][None], k[n, h][None], v[n, h][None],
                                                      beta[n, h][None], la[n, h][None], S[n, h])
            np.testing.assert_allclose(o[n, h], o_ref[0], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(S1[n, h], s_ref, rtol=1e-12, atol=1e-12)


def _pins_hold(mutant):
    """True when every quick pin agrees with the (possibly mutated) oracle."""
    rng = np.random.default_rng(11)
    q, k, v, beta, log_alpha, s0 = _rand_case(rng, 10, 5, 4, gate_mu=0.0)
    checks = []
    o, sT = _run(q, k, v, beta, log_alpha, s0, mutant=mutant)
    o_ref, s_ref = forms.materialised_product(q, k, v, beta, log_alpha, s0)
    checks.append(np.allclose(o, o_ref, rtol=1e-9, atol=1e-10) and np.allclose(sT, s_ref, rtol=1e-9, atol=1e-10))
    o, _ = _run(q, k, v, beta, log_alpha, s0, erase=False, mutant=mutant)
    checks.append(np.allclose(o, forms.gla_closed_form(q, k, v, beta, log_alpha, s0), rtol=1e-9, atol=1e-10))
    o, sT = _run(q, k, v, beta, np.zeros_like(q), s0, mutant=mutant)
    o_ref, s_ref = forms.deltanet_loop_dv_dk(q, k, v, beta, s0)
    checks.append(np.allclose(o, o_ref, rtol=1e-9, atol=1e-10) and np.allclose(sT, s_ref, rtol=1e-9, atol=1e-10))
    return all(checks)


def test_unmutated_oracle_passes_quick_pins():
    assert _pins_hold(None)


@pytest.mark.parametrize("mutant", [1, 2, 3, 4, 5])
def test_mutants_are_caught(mutant):
    """Planted mistakes: 1 read-out before the write, 2 decay after the
    erase, 3 retrieval from the undecayed state, 4 wrong erase sign,
    5 beta dropped from the write."""
    assert not _pins_hold(mutant)


def test_golden_rational_fixture():
    """Stored exact example (tests/golden/kda_rational_d2_t3.json).  Worked by
    hand for the first token: decay gives [[0.5,-1],[1,0.125]], the key
    retrieves (1.1,-0.5), the write vector is 0.5*((1,2)-(1.1,-0.5)) =
    (-0.05,1.25), so S_1 = [[0.47,-0.25],[0.96,1.125]] and o_1 = (0.47,-0.25)."""
    import json
    import os
    from fractions import Fraction
    path = os.path.join(os.path.dirname(__file__), "golden", "kda_rational_d2_t3.json")
    doc = json.load(open(path))
    c = doc["inputs"]
    o, sT = _run(np.array(c["q"], float), np.array(c["k"], float), np.array(c["v"], float),
                 np.array(c["beta"], float), np.log(np.array(c["alpha"], float)),
                 np.array(c["s0"], float))
    want_o = np.array([[float(Fraction(x)) for x in r] for r in doc["o"]])
    want_s = np.array([[float(Fraction(x)) for x in r] for r in doc["final_state"]])
    np.testing.assert_allclose(o[0], [0.47, -0.25], rtol=1e-14)
    np.testing.assert_allclose(o, want_o, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(sT, want_s, rtol=1e-14, atol=1e-15)
