"""GPU parity of the layer variants (the C ABI's KDA_MODE_* flags) against the
fp64 oracle.

- head_gate: one forget gate per (token, head), the scalar gate of "Hybrid
  Linear Attention Architecture: ...", section 3.3.  The oracle takes
  per-channel gates, so it gets the same gate on every key channel.
- erase=False: no erase term, S_t = Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T.
  The oracle's own erase flag gives it.
- normalize_qk / gate_logits: the kernels L2-normalise q, k rows and take gate
  logits (log alpha = -softplus(z)); the oracle gets those inputs computed in
  fp64.

Bars: 2e-2 for bf16 q/k/v, 1e-4 for fp32, as for the plain layer.
"""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_133_b200 as kda
from gated_delta_rule_133_b200.inputs import Workload, cu_from_lengths, draw_tokens, make_inputs
from tests._helpers import TOL_BF16, TOL_F32, f64, norm_max_err

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _head_gates(x):
    """One gate per (token, head): the first channel's gate of the generator."""
    x = dict(x)
    x["log_alpha"] = x["log_alpha"][..., 0].contiguous()
    return x


def _channel_gates(la, d):
    """The oracle's per-channel form of per-head gates."""
    return np.repeat(f64(la)[..., None], d, axis=-1)


@pytest.mark.parametrize("head_gate,erase", [(True, True), (False, False), (True, False)])
@pytest.mark.parametrize("d,dtype", [(128, "bf16"), (64, "bf16"), (128, "fp32")])
def test_chunk_fwd_variants(head_gate, erase, d, dtype):
    B, T, H = 2, 200, 3
    x = make_inputs(Workload("variant", "dense", B, T, H, d, d, dtype, -2.0, 0.05, seed=60 + d), "cpu")
    if head_gate:
        x = _head_gates(x)
    g = {n: (None if t is None else t.to(DEV)) for n, t in x.items()}
    o, sT = kda.kda_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], g["initial_state"],
                              head_gate=head_gate, erase=erase)
    torch.cuda.synchronize()
    kda.kda_check()
    la = _channel_gates(x["log_alpha"], d) if head_gate else f64(x["log_alpha"])
    flat = lambda a: a.reshape(B * T, H, *a.shape[3:])
    o_ref, s_ref = oracle.recurrence(flat(f64(x["q"])), flat(f64(x["k"])), flat(f64(x["v"])),
                                     f64(x["beta"]).reshape(B * T, H), flat(la), np.array([0, T, 2 * T]),
                                     f64(x["initial_state"]), erase=erase)
    tol = TOL_F32 if dtype == "fp32" else TOL_BF16
    assert norm_max_err(f64(o).reshape(B * T, H, d), o_ref) <= tol
    assert norm_max_err(f64(sT), s_ref) <= tol


def test_head_gate_equals_the_same_gate_on_every_channel():
    """The per-head path computes exactly what the per-channel path computes
    when every channel carries the head's gate (same cumsum, same operands)."""
    B, T, H, d = 2, 4 * 64 + 17, 3, 128
    x = _head_gates(make_inputs(Workload("variant", "dense", B, T, H, d, d, "bf16", -2.0, 0.05, seed=63), "cpu"))
    g = {n: (None if t is None else t.to(DEV)) for n, t in x.items()}
    wide = g["log_alpha"].unsqueeze(-1).expand(B, T, H, d).contiguous()
    for erase in (True, False):
        o1, s1 = kda.kda_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], g["initial_state"],
                                   head_gate=True, erase=erase)
        o2, s2 = kda.kda_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], wide, g["initial_state"], erase=erase)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(s1, s2)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_varlen_variants(dtype):
    lens = [1, 63, 130, 0, 65]
    cu = cu_from_lengths(lens)
    x = draw_tokens(int(cu[-1]), 2, 128, 128, dtype, -2.0, 64, "cpu", init_states=len(lens), init_std=0.05)
    x = _head_gates(x)
    g = {n: t.to(DEV) for n, t in x.items()}
    cu_d = torch.from_numpy(cu).to(DEV)
    o, sN = kda.kda_varlen_fwd(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], cu_d, g["initial_state"],
                               head_gate=True, erase=False)
    torch.cuda.synchronize()
    kda.kda_check()
    o_ref, s_ref = oracle.recurrence(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["beta"]),
                                     _channel_gates(x["log_alpha"], 128), cu, f64(x["initial_state"]), erase=False)
    tol = TOL_F32 if dtype == "fp32" else TOL_BF16
    assert norm_max_err(f64(o), o_ref) <= tol
    assert norm_max_err(f64(sN), s_ref) <= tol


@pytest.mark.parametrize("head_gate,erase", [(True, True), (False, False), (True, False)])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_recurrent_step_variants(head_gate, erase, dtype):
    N, H, d, steps = 4, 3, 128, 6
    x = make_inputs(Workload("dec", "decode", N, steps, H, d, d, dtype, -2.0, 0.02, seed=65), "cpu")
    if head_gate:
        x = _head_gates(x)
    state = x["initial_state"].to(DEV).clone()
    S_ref = f64(x["initial_state"])
    tol = TOL_F32 if dtype == "fp32" else TOL_BF16
    for s in range(steps):
        g = {n: x[n][s].to(DEV) for n in ("q", "k", "v", "beta", "log_alpha")}
        o = kda.kda_recurrent_step(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], state,
                                   head_gate=head_gate, erase=erase)
        torch.cuda.synchronize()
        la = _channel_gates(x["log_alpha"][s], d) if head_gate else f64(x["log_alpha"][s])
        o_ref, S_ref = oracle.recurrent_step(f64(x["q"][s]), f64(x["k"][s]), f64(x["v"][s]), f64(x["beta"][s]),
                                             la, S_ref, erase=erase)
        assert norm_max_err(f64(o), o_ref) <= tol
        assert norm_max_err(f64(state), S_ref) <= tol


def _raw(x, seed):
    """Raw projections: q, k rows scaled by random factors (0.2 .. 5) and gate
    logits z with log alpha = -softplus(z) (z ~ N(-3, 1), the generator's)."""
    g = torch.Generator().manual_seed(seed)
    x = dict(x)
    for n in ("q", "k"):
        t = x[n].float()
        scale = torch.exp(torch.empty(*t.shape[:-1], 1).uniform_(-1.6, 1.6, generator=g))
        x[n] = (t * scale).to(x[n].dtype)
    x["log_alpha"] = torch.randn(*x["log_alpha"].shape, generator=g) - 3.0
    return x


def _oracle_inputs(x):
    """What the kernels compute from raw inputs, in fp64: unit rows, -softplus gates."""
    q, k = f64(x["q"]), f64(x["k"])
    q = q / np.maximum(np.linalg.norm(q, axis=-1, keepdims=True), 1e-15)
    k = k / np.maximum(np.linalg.norm(k, axis=-1, keepdims=True), 1e-15)
    z = f64(x["log_alpha"])
    return q, k, -(np.maximum(z, 0) + np.log1p(np.exp(-np.abs(z))))


@pytest.mark.parametrize("d,dtype,head_gate", [(128, "bf16", False), (64, "bf16", False), (128, "bf16", True),
                                               (128, "fp32", False), (128, "fp32", True)])
def test_chunk_fwd_fused_preprocessing(d, dtype, head_gate):
    B, T, H = 2, 200, 3
    x = make_inputs(Workload("variant", "dense", B, T, H, d, d, dtype, -3.0, 0.05, seed=70 + d), "cpu")
    if head_gate:
        x = _head_gates(x)
    x = _raw(x, 71)
    g = {n: (None if t is None else t.to(DEV)) for n, t in x.items()}
    o, sT = kda.kda_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], g["initial_state"],
                              head_gate=head_gate, normalize_qk=True, gate_logits=True)
    torch.cuda.synchronize()
    kda.kda_check()
    q, k, la = _oracle_inputs(x)
    if head_gate:
        la = np.repeat(la[..., None], d, axis=-1)
    flat = lambda a: a.reshape(B * T, H, *a.shape[3:])
    o_ref, s_ref = oracle.recurrence(flat(q), flat(k), flat(f64(x["v"])), f64(x["beta"]).reshape(B * T, H), flat(la),
                                     np.array([0, T, 2 * T]), f64(x["initial_state"]))
    tol = TOL_F32 if dtype == "fp32" else TOL_BF16
    assert norm_max_err(f64(o).reshape(B * T, H, d), o_ref) <= tol
    assert norm_max_err(f64(sT), s_ref) <= tol


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_recurrent_step_fused_preprocessing(dtype):
    N, H, d, steps = 4, 3, 128, 5
    x = _raw(make_inputs(Workload("dec", "decode", N, steps, H, d, d, dtype, -3.0, 0.02, seed=72), "cpu"), 73)
    state = x["initial_state"].to(DEV).clone()
    S_ref = f64(x["initial_state"])
    q, k, la = _oracle_inputs(x)
    tol = TOL_F32 if dtype == "fp32" else TOL_BF16
    for s in range(steps):
        g = {n: x[n][s].to(DEV) for n in ("q", "k", "v", "beta", "log_alpha")}
        o = kda.kda_recurrent_step(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], state,
                                   normalize_qk=True, gate_logits=True)
        torch.cuda.synchronize()
        o_ref, S_ref = oracle.recurrent_step(q[s], k[s], f64(x["v"][s]), f64(x["beta"][s]), la[s], S_ref)
        assert norm_max_err(f64(o), o_ref) <= tol
        assert norm_max_err(f64(state), S_ref) <= tol


def test_varlen_fused_preprocessing():
    lens = [5, 130, 64]
    cu = cu_from_lengths(lens)
    x = _raw(draw_tokens(int(cu[-1]), 2, 128, 128, "bf16", -3.0, 74, "cpu", init_states=len(lens), init_std=0.05), 75)
    g = {n: t.to(DEV) for n, t in x.items()}
    o, sN = kda.kda_varlen_fwd(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], torch.from_numpy(cu).to(DEV),
                               g["initial_state"], normalize_qk=True, gate_logits=True)
    torch.cuda.synchronize()
    kda.kda_check()
    q, k, la = _oracle_inputs(x)
    o_ref, s_ref = oracle.recurrence(q, k, f64(x["v"]), f64(x["beta"]), la, cu, f64(x["initial_state"]))
    assert norm_max_err(f64(o), o_ref) <= TOL_BF16
    assert norm_max_err(f64(sN), s_ref) <= TOL_BF16
