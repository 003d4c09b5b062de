"""Parity at the full sizes of the four large workloads, in the same launch
configuration the benchmark times.  The GPU runs the whole workload; the fp64
oracle recomputes a sample it can finish in seconds (a subset of heads, all
their tokens; the long-context case compares every 97th token plus the final
states; decode compares a subset of sequences at every step)."""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_133_b200 as kda
from gated_delta_rule_133_b200.inputs import WORKLOADS, make_inputs
from tests._helpers import TOL_BF16, f64, norm_max_err

pytestmark = pytest.mark.gpu


def _heads_f64(x, heads, axis):
    return f64(torch.index_select(x, axis, torch.tensor(heads, device=x.device)))


def test_prefill_full():
    w = WORKLOADS["prefill"]
    d = make_inputs(w, "cuda")
    o, sT = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["log_alpha"], d["initial_state"])
    torch.cuda.synchronize()
    kda.kda_check()
    heads = [0, 5, 10, 15]
    B, T = w.B, w.T
    flat = lambda x: _heads_f64(x, heads, 2).reshape(B * T, len(heads), *x.shape[3:])
    o_ref, s_ref = oracle.recurrence(flat(d["q"]), flat(d["k"]), flat(d["v"]),
                                     _heads_f64(d["beta"], heads, 2).reshape(B * T, len(heads)),
                                     flat(d["log_alpha"]), np.array([0, T, 2 * T]),
                                     _heads_f64(d["initial_state"], heads, 1))
    assert norm_max_err(flat(o), o_ref) <= TOL_BF16
    assert norm_max_err(_heads_f64(sT, heads, 1), s_ref) <= TOL_BF16
    assert torch.isfinite(o).all() and torch.isfinite(sT).all()


def test_varlen_full():
    w = WORKLOADS["varlen"]
    d = make_inputs(w, "cuda")
    o, sN = kda.kda_varlen_fwd(d["q"], d["k"], d["v"], d["beta"], d["log_alpha"], d["cu_seqlens"], None)
    torch.cuda.synchronize()
    kda.kda_check()
    heads = [3, 17]
    cu = d["cu_seqlens"].cpu().numpy()
    o_ref, s_ref = oracle.recurrence(_heads_f64(d["q"], heads, 1), _heads_f64(d["k"], heads, 1),
                                     _heads_f64(d["v"], heads, 1), _heads_f64(d["beta"], heads, 1),
                                     _heads_f64(d["log_alpha"], heads, 1), cu, None)
    assert norm_max_err(_heads_f64(o, heads, 1), o_ref) <= TOL_BF16
    assert norm_max_err(_heads_f64(sN, heads, 1), s_ref) <= TOL_BF16
    assert torch.isfinite(o).all() and torch.isfinite(sN).all()


def test_long_context_full():
    w = WORKLOADS["long"]
    d = make_inputs(w, "cuda")
    o, sT = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["log_alpha"], None)
    torch.cuda.synchronize()
    kda.kda_check()
    heads = [1, 30]
    sq = lambda x: _heads_f64(x[0], heads, 1)
    o_ref, s_ref = oracle.recurrence(sq(d["q"]), sq(d["k"]), sq(d["v"]), sq(d["beta"]), sq(d["log_alpha"]))
    idx = np.arange(0, w.T, 97)
    assert norm_max_err(sq(o)[idx], o_ref[idx]) <= TOL_BF16
    assert norm_max_err(_heads_f64(sT, heads, 1), s_ref) <= TOL_BF16
    assert torch.isfinite(o).all() and torch.isfinite(sT).all()


def test_decode_full():
    w = WORKLOADS["decode"]
    x = make_inputs(w, "cuda")
    state = x["initial_state"].clone()
    seqs = [0, 77, 255]
    pick = lambda t: _heads_f64(t, seqs, 0)
    S_ref = pick(x["initial_state"])
    for s in range(w.T):
        o = kda.kda_recurrent_step(x["q"][s], x["k"][s], x["v"][s], x["beta"][s], x["log_alpha"][s], state)
        torch.cuda.synchronize()
        o_ref, S_ref = oracle.recurrent_step(pick(x["q"][s]), pick(x["k"][s]), pick(x["v"][s]),
                                             pick(x["beta"][s]), pick(x["log_alpha"][s]), S_ref)
        assert norm_max_err(pick(o), o_ref) <= TOL_BF16
    kda.kda_check()
    assert norm_max_err(pick(state), S_ref) <= TOL_BF16
    assert torch.isfinite(state).all()


@pytest.mark.parametrize("variant", ["head_gate", "no_erase"])
def test_prefill_variants_full(variant):
    """The two gate tiers on the full prefill workload (the bench's
    prefill_head_gate / prefill_no_erase lines), four heads against the
    oracle (the per-head gate given on every channel; the erase flag off)."""
    w = WORKLOADS["prefill"]
    d = make_inputs(w, "cuda")
    la = d["log_alpha"]
    kw = {}
    if variant == "head_gate":
        la = la[..., 0].contiguous()
        kw["head_gate"] = True
    else:
        kw["erase"] = False
    o, sT = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], la, d["initial_state"], **kw)
    torch.cuda.synchronize()
    kda.kda_check()
    heads = [1, 6, 11, 14]
    B, T = w.B, w.T
    flat = lambda x: _heads_f64(x, heads, 2).reshape(B * T, len(heads), *x.shape[3:])
    la_ref = flat(d["log_alpha"]) if variant == "no_erase" else \
        np.repeat(_heads_f64(la, heads, 2).reshape(B * T, len(heads), 1), w.dk, axis=2)
    o_ref, s_ref = oracle.recurrence(flat(d["q"]), flat(d["k"]), flat(d["v"]),
                                     _heads_f64(d["beta"], heads, 2).reshape(B * T, len(heads)),
                                     la_ref, np.array([0, T, 2 * T]), _heads_f64(d["initial_state"], heads, 1),
                                     erase=variant != "no_erase")
    assert norm_max_err(flat(o), o_ref) <= TOL_BF16
    assert norm_max_err(_heads_f64(sT, heads, 1), s_ref) <= TOL_BF16


def test_dplr_prefill_full():
    """The diagonal-plus-low-rank forward on the prefill workload with the
    bench's a, b draw (seed 11), two whole (sequence, head) pairs against the
    oracle's token recurrence."""
    from oracle import dplr
    w = WORKLOADS["prefill"]
    d = make_inputs(w, "cuda")
    g = torch.Generator(device="cuda").manual_seed(11)
    a, b = [(torch.randn(w.B, w.T, w.H, w.dk, generator=g, device="cuda") * 0.7 / w.dk ** 0.5).to(torch.bfloat16)
            for _ in range(2)]
    o, sT = kda.kda_dplr_fwd(d["q"], d["k"], d["v"], a, b, d["log_alpha"], d["initial_state"])
    torch.cuda.synchronize()
    kda.kda_check()
    for n, h in ((0, 2), (1, 13)):
        sl = lambda x: f64(x[n, :, h:h + 1])
        o_ref, s_ref = dplr.recurrence(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(a), sl(b), sl(d["log_alpha"]), None,
                                       f64(d["initial_state"][n:n + 1, h:h + 1]))
        assert norm_max_err(sl(o), o_ref) <= 1e-4
        assert norm_max_err(f64(sT[n:n + 1, h:h + 1]), s_ref) <= 1e-4
