"""GPU: packed batches of many variable-length sequences, the device-side
boundary guard, and the caller-provided workspace.

The scan order of a packed batch (longest sequence first) is computed once per
call on the device; these cases cover a thousand sequences (lengths 0, 1, 63,
64, 65 among them), and more sequences than the sort keeps in shared memory.
"""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_133_b200 as kda
from gated_delta_rule_133_b200.inputs import cu_from_lengths, draw_tokens
from tests._helpers import TOL_BF16, f64, norm_max_err

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _case(lens, H, d, seed, with_s0=True):
    cu = cu_from_lengths(lens)
    t = draw_tokens(int(cu[-1]), H, d, d, "bf16", -3.0, seed, "cpu", init_states=len(lens), init_std=0.05)
    t["cu_seqlens"] = torch.from_numpy(cu)
    if not with_s0:
        t["initial_state"] = None
    return t


def _gpu(t):
    return {k: (None if v is None else v.to(DEV)) for k, v in t.items()}


def _oracle(t):
    return oracle.recurrence(f64(t["q"]), f64(t["k"]), f64(t["v"]), f64(t["beta"]), f64(t["log_alpha"]),
                             t["cu_seqlens"].numpy(), f64(t["initial_state"]))


def _lengths(n, seed, hi=200):
    rng = np.random.default_rng(seed)
    lens = list(rng.integers(0, hi, size=n))
    for i, L in enumerate((0, 1, 63, 64, 65, 0, 128, 129)):   # the edge lengths, spread over the batch
        lens[(i * 131) % n] = L
    return [int(x) for x in lens]


@pytest.mark.parametrize("with_s0", [True, False])
def test_thousand_sequences_match_oracle(with_s0):
    lens = _lengths(1000, 5 + with_s0)
    t = _case(lens, 2, 128, 80 + with_s0, with_s0)
    g = _gpu(t)
    o, sN = kda.kda_varlen_fwd(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], g["cu_seqlens"],
                               g["initial_state"])
    torch.cuda.synchronize()
    kda.kda_check()
    o_ref, s_ref = _oracle(t)
    assert norm_max_err(f64(o), o_ref) <= TOL_BF16
    assert norm_max_err(f64(sN), s_ref) <= TOL_BF16
    empty = [i for i, L in enumerate(lens) if L == 0]
    for i in empty:   # empty sequences pass their initial state (or zeros) through
        want = g["initial_state"][i] if with_s0 else torch.zeros_like(sN[i])
        assert torch.equal(sN[i], want)


def test_more_sequences_than_the_shared_memory_sort():
    """20000 short sequences: the longest-first order is sorted in the workspace."""
    rng = np.random.default_rng(9)
    lens = [int(x) for x in rng.integers(0, 5, size=20000)]
    lens[17] = 130
    t = _case(lens, 1, 64, 91)
    g = _gpu(t)
    o, sN = kda.kda_varlen_fwd(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], g["cu_seqlens"],
                               g["initial_state"])
    torch.cuda.synchronize()
    kda.kda_check()
    o_ref, s_ref = _oracle(t)
    assert norm_max_err(f64(o), o_ref) <= TOL_BF16
    assert norm_max_err(f64(sN), s_ref) <= TOL_BF16


@pytest.mark.parametrize("cuda_cores", [False, True])
def test_boundaries_outside_the_tokens_are_skipped_and_reported(cuda_cores):
    """cu_seqlens whose last sequence runs past the token axis: that sequence
    is skipped (o rows untouched, final state = initial state), the others are
    computed, and kda_check reports KDA_ERR_INVALID_ARG once."""
    lens = [100, 150, 50]
    t = _case(lens, 2, 128, 93)
    g = _gpu(t)
    T = 300
    bad_cu = torch.tensor([0, 100, 250, 400], dtype=torch.int32, device=DEV)
    o = torch.full((T, 2, 128), float("nan"), device=DEV)
    o, sN = kda.kda_varlen_fwd(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], bad_cu, g["initial_state"],
                               o=o, cuda_cores=cuda_cores)
    torch.cuda.synchronize()
    with pytest.raises(kda.KdaError) as e:
        kda.kda_check()
    assert e.value.status == kda._lib.KDA_ERR_INVALID_ARG
    kda.kda_check()   # the status word was cleared
    o_ref, s_ref = _oracle(t)
    assert norm_max_err(f64(o[:250]), o_ref[:250]) <= TOL_BF16
    assert norm_max_err(f64(sN[:2]), s_ref[:2]) <= TOL_BF16
    assert torch.isnan(o[250:]).all()
    assert torch.equal(sN[2], g["initial_state"][2])


def test_dirty_caller_workspace_gives_identical_results():
    """A caller's workspace full of garbage gives bit-identical results to a
    fresh one: the library initialises what it needs (hand-off flags)."""
    from gated_delta_rule_133_b200.inputs import Workload, make_inputs
    w = Workload("ws", "dense", 2, 700, 4, 128, 128, "bf16", -3.0, 0.05, seed=94)
    g = _gpu(make_inputs(w, "cpu"))
    args = (g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], g["initial_state"])
    o1, s1 = kda.kda_chunk_fwd(*args)
    n = kda.chunk_fwd_workspace_size(2, 700, 4, 128, 128)
    ws = torch.full((n + 4096,), 0xFF, dtype=torch.uint8, device=DEV)
    o2, s2 = kda.kda_chunk_fwd(*args, workspace=ws)
    o3, s3 = kda.kda_chunk_fwd(*args, workspace=ws)   # reused as it was left
    t = _case([300, 1, 0, 257], 2, 128, 95)
    v = _gpu(t)
    vargs = (v["q"], v["k"], v["v"], v["beta"], v["log_alpha"], v["cu_seqlens"], v["initial_state"])
    vo1, vs1 = kda.kda_varlen_fwd(*vargs)
    nv = kda.varlen_fwd_workspace_size(4, 558, 2, 128, 128)
    vws = torch.full((nv,), 0xFF, dtype=torch.uint8, device=DEV)
    vo2, vs2 = kda.kda_varlen_fwd(*vargs, workspace=vws)
    torch.cuda.synchronize()
    kda.kda_check()
    assert torch.equal(o1, o2) and torch.equal(s1, s2) and torch.equal(o1, o3) and torch.equal(s1, s3)
    assert torch.equal(vo1, vo2) and torch.equal(vs1, vs2)
