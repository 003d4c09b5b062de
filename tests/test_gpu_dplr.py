"""GPU: the diagonal-plus-low-rank transition (kda_dplr_fwd / kda_dplr_varlen_fwd
through the C ABI) against the fp64 oracle (oracle.dplr.recurrence).

The kernel computes in fp32 from the exact input values: bar 1e-4 (max-abs
error / RMS of the reference), as for the fp32 layer.  Low-rank vectors a, b
are drawn at the scale that keeps the transition's spectral radius near one
(a, b ~ N(0, s^2 / d_k)).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import dplr
import gated_delta_rule_133_b200 as kda
from gated_delta_rule_133_b200.inputs import cu_from_lengths, draw_tokens
from tests._helpers import f64, norm_max_err

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOL = 1e-4


def _ab(T, H, dk, dtype, seed, scale=0.7):
    g = torch.Generator().manual_seed(seed)
    t = torch.float32 if dtype == "fp32" else torch.bfloat16
    a = (torch.randn(T, H, dk, generator=g) * scale / dk ** 0.5).to(t)
    b = (torch.randn(T, H, dk, generator=g) * scale / dk ** 0.5).to(t)
    return a, b


@pytest.mark.parametrize("T,d,dtype,mu", [(150, 128, "bf16", -3.0), (64, 64, "fp32", -1.0), (1, 128, "bf16", -3.0),
                                          (200, 64, "bf16", -6.0)])
def test_dplr_dense_matches_oracle(T, d, dtype, mu):
    B, H = 2, 2
    x = draw_tokens(B * T, H, d, d, dtype, mu, 500 + T, "cpu", init_states=B, init_std=0.05)
    a, b = _ab(B * T, H, d, dtype, 600 + T)
    shape = lambda t: t.reshape(B, T, *t.shape[1:]).to(DEV)
    o, sT = kda.kda_dplr_fwd(shape(x["q"]), shape(x["k"]), shape(x["v"]), shape(a), shape(b),
                             shape(x["log_alpha"]), x["initial_state"].to(DEV))
    torch.cuda.synchronize()
    kda.kda_check()
    o_ref, s_ref = dplr.recurrence(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(a), f64(b), f64(x["log_alpha"]),
                                   np.arange(B + 1) * T, f64(x["initial_state"]))
    assert norm_max_err(f64(o).reshape(B * T, H, d), o_ref) <= TOL
    assert norm_max_err(f64(sT), s_ref) <= TOL


def test_dplr_with_kda_vectors_is_the_layer():
    """a = alpha k, b = -beta k, key beta k: the KDA layer's result (fp32 path)."""
    B, T, H, d = 1, 130, 2, 64
    x = draw_tokens(T, H, d, d, "fp32", -2.0, 510, "cpu", init_states=1, init_std=0.05)
    beta = x["beta"][..., None]
    a = torch.exp(x["log_alpha"]) * x["k"]
    b = -beta * x["k"]
    kb = beta * x["k"]
    g = lambda t: t.unsqueeze(0).contiguous().to(DEV)
    o, sT = kda.kda_dplr_fwd(g(x["q"]), g(kb), g(x["v"]), g(a), g(b), g(x["log_alpha"]), x["initial_state"].to(DEV))
    o2, s2 = kda.kda_chunk_fwd(g(x["q"]), g(x["k"]), g(x["v"]), g(x["beta"]), g(x["log_alpha"]),
                               x["initial_state"].to(DEV))
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.recurrence(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["beta"]), f64(x["log_alpha"]),
                                     np.array([0, T]), f64(x["initial_state"]))
    assert norm_max_err(f64(o)[0], o_ref) <= TOL and norm_max_err(f64(sT), s_ref) <= TOL
    assert norm_max_err(f64(o2)[0], o_ref) <= TOL


def test_dplr_varlen_matches_oracle():
    lens = [1, 63, 64, 65, 0, 200]
    cu = cu_from_lengths(lens)
    H, d = 2, 128
    x = draw_tokens(int(cu[-1]), H, d, d, "bf16", -3.0, 520, "cpu", init_states=len(lens), init_std=0.05)
    a, b = _ab(int(cu[-1]), H, d, "bf16", 521)
    o, sN = kda.kda_dplr_varlen_fwd(x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV), a.to(DEV), b.to(DEV),
                                    x["log_alpha"].to(DEV), torch.from_numpy(cu).to(DEV), x["initial_state"].to(DEV))
    torch.cuda.synchronize()
    kda.kda_check()
    o_ref, s_ref = dplr.recurrence(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(a), f64(b), f64(x["log_alpha"]), cu,
                                   f64(x["initial_state"]))
    assert norm_max_err(f64(o), o_ref) <= TOL
    assert norm_max_err(f64(sN), s_ref) <= TOL


def test_dplr_varlen_boundaries_outside_the_tokens_are_skipped_and_reported():
    """cu_seqlens whose last sequence runs past the token axis: that sequence
    is skipped (o rows untouched, final state = initial state), the others are
    computed, and kda_check reports KDA_ERR_INVALID_ARG."""
    lens = [100, 150, 50]
    cu = cu_from_lengths(lens)
    H, d, T = 2, 128, 300
    x = draw_tokens(T, H, d, d, "bf16", -3.0, 530, "cpu", init_states=3, init_std=0.05)
    a, b = _ab(T, H, d, "bf16", 531)
    s0 = x["initial_state"].to(DEV)
    o = torch.full((T, H, d), float("nan"), device=DEV)
    bad_cu = torch.tensor([0, 100, 250, 400], dtype=torch.int32, device=DEV)
    o, sN = kda.kda_dplr_varlen_fwd(x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV), a.to(DEV), b.to(DEV),
                                    x["log_alpha"].to(DEV), bad_cu, s0, o=o)
    torch.cuda.synchronize()
    with pytest.raises(kda.KdaError) as e:
        kda.kda_check()
    assert e.value.status == kda._lib.KDA_ERR_INVALID_ARG
    o_ref, s_ref = dplr.recurrence(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(a), f64(b), f64(x["log_alpha"]), cu,
                                   f64(x["initial_state"]))
    assert norm_max_err(f64(o[:250]), o_ref[:250]) <= TOL
    assert norm_max_err(f64(sN[:2]), s_ref[:2]) <= TOL
    assert torch.isnan(o[250:]).all()
    assert torch.equal(sN[2], s0[2])


def test_dplr_dirty_workspace_gives_identical_results():
    """A caller workspace full of garbage gives bit-identical results."""
    B, T, H, d = 2, 300, 2, 128
    x = draw_tokens(B * T, H, d, d, "bf16", -3.0, 540, "cpu", init_states=B, init_std=0.05)
    a, b = _ab(B * T, H, d, "bf16", 541)
    r = lambda t: t.reshape(B, T, *t.shape[1:]).to(DEV)
    args = (r(x["q"]), r(x["k"]), r(x["v"]), r(a), r(b), r(x["log_alpha"]), x["initial_state"].to(DEV))
    o1, s1 = kda.kda_dplr_fwd(*args)
    ws = torch.full((kda.dplr_fwd_workspace_size(B, T, H, d, d),), 0xFF, dtype=torch.uint8, device=DEV)
    o2, s2 = kda.kda_dplr_fwd(*args, workspace=ws)
    torch.cuda.synchronize()
    kda.kda_check()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


def test_dplr_bf16_output_is_the_rounded_fp32_output():
    """o_dtype=bf16 stores exactly the fp32 result rounded to nearest even."""
    B, T, H, d = 1, 200, 2, 128
    x = draw_tokens(B * T, H, d, d, "bf16", -3.0, 550, "cpu", init_states=B, init_std=0.05)
    a, b = _ab(B * T, H, d, "bf16", 551)
    r = lambda t: t.reshape(B, T, *t.shape[1:]).to(DEV)
    args = (r(x["q"]), r(x["k"]), r(x["v"]), r(a), r(b), r(x["log_alpha"]), x["initial_state"].to(DEV))
    o32, s32 = kda.kda_dplr_fwd(*args)
    o16, s16 = kda.kda_dplr_fwd(*args, o_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    kda.kda_check()
    assert o16.dtype == torch.bfloat16 and torch.equal(o16, o32.to(torch.bfloat16))
    assert torch.equal(s16, s32)


def test_dplr_many_packed_sequences():
    """Several hundred packed sequences, lengths 0, 1, 63, 64 and 65 among them."""
    rng = np.random.default_rng(560)
    lens = [int(x) for x in rng.integers(0, 150, size=300)]
    for i, L in enumerate((0, 1, 63, 64, 65, 128, 129)):
        lens[(i * 41) % len(lens)] = L
    cu = cu_from_lengths(lens)
    H, d = 2, 64
    x = draw_tokens(int(cu[-1]), H, d, d, "bf16", -3.0, 561, "cpu", init_states=len(lens), init_std=0.05)
    a, b = _ab(int(cu[-1]), H, d, "bf16", 562)
    o, sN = kda.kda_dplr_varlen_fwd(x["q"].to(DEV), x["k"].to(DEV), x["v"].to(DEV), a.to(DEV), b.to(DEV),
                                    x["log_alpha"].to(DEV), torch.from_numpy(cu).to(DEV), x["initial_state"].to(DEV))
    torch.cuda.synchronize()
    kda.kda_check()
    o_ref, s_ref = dplr.recurrence(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(a), f64(b), f64(x["log_alpha"]), cu,
                                   f64(x["initial_state"]))
    assert norm_max_err(f64(o), o_ref) <= TOL
    assert norm_max_err(f64(sN), s_ref) <= TOL
