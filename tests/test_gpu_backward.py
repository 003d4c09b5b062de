"""GPU: the chunkwise backward (kda_chunk_bwd / kda_varlen_bwd through the C
ABI) against the fp64 oracle's reverse-mode gradients of the token recurrence
(oracle.backward.recurrence_backward, itself pinned by finite differences).

The kernel computes in fp32 from the exact input values; the bar is 1e-4
(max-abs error / RMS of the reference, per gradient), the fp32 forward's bar.
"""
import numpy as np
import pytest
import torch

from oracle import backward
import gated_delta_rule_133_b200 as kda
from gated_delta_rule_133_b200.inputs import Workload, cu_from_lengths, draw_tokens, make_inputs
from tests._helpers import f64, norm_max_err

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOL = 1e-4
NAMES = ("dq", "dk", "dv", "dbeta", "dlog_alpha", "ds0")


def _grads_out(B, T, H, dv, seed):
    g = torch.Generator().manual_seed(seed)
    do = torch.randn(B, T, H, dv, generator=g)
    dsT = torch.randn(B, H, 128 if dv == 128 else dv, dv, generator=g)
    return do, dsT


def _check(got, ref):
    for n, a, b in zip(NAMES, got, ref):
        e = norm_max_err(a, b)
        assert e <= TOL, f"{n}: {e:.2e}"


@pytest.mark.parametrize("B,T,H,d,dtype,mu", [
    (2, 150, 2, 128, "bf16", -3.0),     # two full chunks and a ragged one
    (1, 64, 3, 64, "fp32", -1.0),       # one full chunk, strong gates
    (1, 1, 2, 128, "bf16", -3.0),       # a single token
    (2, 200, 1, 64, "bf16", -6.0),      # weak gates
])
def test_chunk_bwd_matches_oracle(B, T, H, d, dtype, mu):
    w = Workload("bwd", "dense", B, T, H, d, d, dtype, mu, 0.05, seed=300 + T)
    x = make_inputs(w, "cpu")
    g = torch.Generator().manual_seed(400 + T)
    do = torch.randn(B, T, H, d, generator=g)
    dsT = torch.randn(B, H, d, d, generator=g)
    dev = {n: (None if t is None else t.to(DEV)) for n, t in x.items()}
    got = kda.kda_chunk_bwd(dev["q"], dev["k"], dev["v"], dev["beta"], dev["log_alpha"], dev["initial_state"],
                            do.to(DEV), dsT.to(DEV))
    torch.cuda.synchronize()
    kda.kda_check()
    flat = lambda t: f64(t).reshape(B * T, H, *t.shape[3:])
    ref = backward.recurrence_backward(flat(x["q"]), flat(x["k"]), flat(x["v"]), f64(x["beta"]).reshape(B * T, H),
                                       flat(x["log_alpha"]), np.arange(B + 1) * T, f64(x["initial_state"]),
                                       flat(do), f64(dsT))
    got = [flat(t) for t in got[:5]] + [f64(got[5])]
    got[3] = got[3].reshape(B * T, H)
    _check(got, ref)


def test_chunk_bwd_without_state_gradients():
    """No initial state and no final-state gradient: both read as zeros."""
    B, T, H, d = 1, 130, 2, 128
    w = Workload("bwd", "dense", B, T, H, d, d, "bf16", -3.0, 0.0, seed=310)
    x = make_inputs(w, "cpu")
    do = torch.randn(B, T, H, d, generator=torch.Generator().manual_seed(311))
    dev = {n: (None if t is None else t.to(DEV)) for n, t in x.items()}
    got = kda.kda_chunk_bwd(dev["q"], dev["k"], dev["v"], dev["beta"], dev["log_alpha"], None, do.to(DEV), None)
    torch.cuda.synchronize()
    flat = lambda t: f64(t).reshape(B * T, H, *t.shape[3:])
    ref = backward.recurrence_backward(flat(x["q"]), flat(x["k"]), flat(x["v"]), f64(x["beta"]).reshape(B * T, H),
                                       flat(x["log_alpha"]), None, None, flat(do), None)
    got = [flat(t) for t in got[:5]] + [f64(got[5])]
    got[3] = got[3].reshape(B * T, H)
    _check(got, ref)


def test_varlen_bwd_matches_oracle():
    lens = [1, 63, 64, 65, 0, 200, 129]
    cu = cu_from_lengths(lens)
    H, d = 2, 128
    t = draw_tokens(int(cu[-1]), H, d, d, "bf16", -3.0, 320, "cpu", init_states=len(lens), init_std=0.05)
    g = torch.Generator().manual_seed(321)
    do = torch.randn(int(cu[-1]), H, d, generator=g)
    dsT = torch.randn(len(lens), H, d, d, generator=g)
    dev = {n: (None if v is None else v.to(DEV)) for n, v in t.items()}
    got = kda.kda_varlen_bwd(dev["q"], dev["k"], dev["v"], dev["beta"], dev["log_alpha"],
                             torch.from_numpy(cu).to(DEV), dev["initial_state"], do.to(DEV), dsT.to(DEV))
    torch.cuda.synchronize()
    kda.kda_check()
    ref = backward.recurrence_backward(f64(t["q"]), f64(t["k"]), f64(t["v"]), f64(t["beta"]), f64(t["log_alpha"]),
                                       cu, f64(t["initial_state"]), f64(do), f64(dsT))
    _check([f64(x) for x in got], ref)


def test_chunk_bwd_prefill_shape_sampled_heads():
    """The prefill workload at full size (B2 H16 T4096, bf16), gradients of two
    whole (sequence, head) pairs against the oracle (heads are independent)."""
    from gated_delta_rule_133_b200.inputs import WORKLOADS
    w = WORKLOADS["prefill"]
    x = make_inputs(w, DEV)
    g = torch.Generator(device=DEV).manual_seed(330)
    do = torch.randn(w.B, w.T, w.H, w.dv, generator=g, device=DEV)
    dsT = torch.randn(w.B, w.H, w.dk, w.dv, generator=g, device=DEV)
    got = kda.kda_chunk_bwd(x["q"], x["k"], x["v"], x["beta"], x["log_alpha"], x["initial_state"], do, dsT)
    torch.cuda.synchronize()
    kda.kda_check()
    for n, h in ((0, 3), (1, 12)):
        sl = lambda t: f64(t[n, :, h:h + 1])
        ref = backward.recurrence_backward(sl(x["q"]), sl(x["k"]), sl(x["v"]), f64(x["beta"][n, :, h:h + 1]),
                                           sl(x["log_alpha"]), None, f64(x["initial_state"][n:n + 1, h:h + 1]),
                                           sl(do), f64(dsT[n:n + 1, h:h + 1]))
        mine = [sl(t) for t in got[:3]] + [f64(got[3][n, :, h:h + 1]), sl(got[4]),
                                            f64(got[5][n:n + 1, h:h + 1])]
        _check(mine, ref)


def test_varlen_bwd_boundaries_outside_the_tokens_are_skipped_and_reported():
    """cu_seqlens whose last sequence runs past the token axis: that sequence
    is skipped (zero gradients for its rows, dS_0 = dS_T), the others match
    the oracle, and kda_check reports KDA_ERR_INVALID_ARG."""
    lens = [100, 150, 50]
    cu = cu_from_lengths(lens)
    H, d, T = 2, 128, 300
    t = draw_tokens(T, H, d, d, "bf16", -3.0, 340, "cpu", init_states=3, init_std=0.05)
    g = torch.Generator().manual_seed(341)
    do = torch.randn(T, H, d, generator=g)
    dsT = torch.randn(3, H, d, d, generator=g)
    dev = {n: (None if v is None else v.to(DEV)) for n, v in t.items()}
    bad_cu = torch.tensor([0, 100, 250, 400], dtype=torch.int32, device=DEV)
    got = kda.kda_varlen_bwd(dev["q"], dev["k"], dev["v"], dev["beta"], dev["log_alpha"], bad_cu,
                             dev["initial_state"], do.to(DEV), dsT.to(DEV))
    torch.cuda.synchronize()
    with pytest.raises(kda.KdaError) as e:
        kda.kda_check()
    assert e.value.status == kda._lib.KDA_ERR_INVALID_ARG
    n = 250
    ref = backward.recurrence_backward(f64(t["q"])[:n], f64(t["k"])[:n], f64(t["v"])[:n], f64(t["beta"])[:n],
                                       f64(t["log_alpha"])[:n], cu[:3], f64(t["initial_state"])[:2],
                                       f64(do)[:n], f64(dsT)[:2])
    _check([f64(x)[:n] for x in got[:5]] + [f64(got[5])[:2]], ref)
    for x in (got[0], got[1], got[3], got[4]):
        assert not x[n:].any()
    assert torch.equal(got[5][2], dsT[2].to(DEV))


def test_bwd_dirty_workspace_gives_identical_results():
    """A caller workspace full of garbage gives bit-identical gradients."""
    B, T, H, d = 2, 200, 2, 128
    w = Workload("bwd", "dense", B, T, H, d, d, "bf16", -3.0, 0.05, seed=350)
    x = {n: (None if v is None else v.to(DEV)) for n, v in make_inputs(w, "cpu").items()}
    do = torch.randn(B, T, H, d, generator=torch.Generator().manual_seed(351)).to(DEV)
    args = (x["q"], x["k"], x["v"], x["beta"], x["log_alpha"], x["initial_state"], do)
    g1 = kda.kda_chunk_bwd(*args)
    n = kda._lib.workspace_size("kda_chunk_bwd_workspace_size", B, T, H, d, d, 64, kda._lib.KDA_BF16)
    ws = torch.full((n,), 0xFF, dtype=torch.uint8, device=DEV)
    g2 = kda.kda_chunk_bwd(*args, workspace=ws)
    torch.cuda.synchronize()
    kda.kda_check()
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def test_varlen_bwd_many_packed_sequences():
    """Several hundred packed sequences, lengths 0, 1, 63, 64 and 65 among them."""
    rng = np.random.default_rng(360)
    lens = [int(x) for x in rng.integers(0, 150, size=300)]
    for i, L in enumerate((0, 1, 63, 64, 65, 128, 129)):
        lens[(i * 41) % len(lens)] = L
    cu = cu_from_lengths(lens)
    H, d = 2, 64
    t = draw_tokens(int(cu[-1]), H, d, d, "bf16", -3.0, 361, "cpu", init_states=len(lens), init_std=0.05)
    g = torch.Generator().manual_seed(362)
    do = torch.randn(int(cu[-1]), H, d, generator=g)
    dsT = torch.randn(len(lens), H, d, d, generator=g)
    dev = {n: (None if v is None else v.to(DEV)) for n, v in t.items()}
    got = kda.kda_varlen_bwd(dev["q"], dev["k"], dev["v"], dev["beta"], dev["log_alpha"],
                             torch.from_numpy(cu).to(DEV), dev["initial_state"], do.to(DEV), dsT.to(DEV))
    torch.cuda.synchronize()
    kda.kda_check()
    ref = backward.recurrence_backward(f64(t["q"]), f64(t["k"]), f64(t["v"]), f64(t["beta"]), f64(t["log_alpha"]),
                                       cu, f64(t["initial_state"]), f64(do), f64(dsT))
    _check([f64(x) for x in got], ref)
