"""GPU: the two-stream blocked schedule of the tensor-core chunk forward.

For dense inputs the library splits the chunk axis into blocks: the prep pass
of block b + 1 runs on a second stream while block b is scanned, and the state
crosses block boundaries through memory as the same fp32 values it has in
registers.  Every block count (KDA_MODE_BLOCKS(n), the ``blocks`` keyword)
must therefore give results bit-identical to the single-block schedule, which
itself matches the oracle.
"""

import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_133_b200 as kda
from gated_delta_rule_133_b200.inputs import Workload, make_inputs
from tests._helpers import TOL_BF16, f64, norm_max_err

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _inputs(B, T, H, d, seed, init=0.05):
    w = Workload("blocked", "dense", B, T, H, d, d, "bf16", -3.0, init, seed=seed)
    x = make_inputs(w, "cpu")
    return x, {k: (None if v is None else v.to(DEV)) for k, v in x.items()}


def _call(g, blocks, initial_state="inputs", **kw):
    s0 = g["initial_state"] if isinstance(initial_state, str) else initial_state
    out = kda.kda_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], s0, blocks=blocks, **kw)
    torch.cuda.synchronize()
    kda.kda_check()
    return out


@pytest.mark.parametrize("d", [128, 64])
def test_block_counts_bit_identical(d):
    """T = 33 chunks + a ragged tail: even, uneven and empty trailing blocks."""
    x, g = _inputs(2, 33 * 64 + 37, 3, d, seed=41)
    o1, s1 = _call(g, 1)
    for nb in (2, 3, 5, 8):
        o, s = _call(g, nb)
        assert torch.equal(o, o1), nb
        assert torch.equal(s, s1), nb
    # and the single-block result is the oracle's
    B, T, H = x["q"].shape[:3]
    flat = lambda t: f64(t).reshape(B * T, H, *t.shape[3:])
    o_ref, s_ref = oracle.recurrence(flat(x["q"]), flat(x["k"]), flat(x["v"]), f64(x["beta"]).reshape(B * T, H),
                                     flat(x["log_alpha"]), np.arange(B + 1) * T, f64(x["initial_state"]))
    assert norm_max_err(f64(o1).reshape(B * T, H, d), o_ref) <= TOL_BF16
    assert norm_max_err(f64(s1), s_ref) <= TOL_BF16


def test_blocked_without_final_state():
    """No final state requested: the carry lives in the workspace."""
    x, g = _inputs(2, 40 * 64, 2, 128, seed=42)
    o1, _ = _call(g, 1)
    o4, s4 = _call(g, 4, output_final_state=False)
    assert s4 is None
    assert torch.equal(o4, o1)


def test_blocked_in_place_state():
    """initial_state and final_state the same buffer, several blocks."""
    x, g = _inputs(1, 48 * 64, 2, 128, seed=43)
    o1, s1 = _call(g, 1)
    st = g["initial_state"].clone()
    o3, _ = _call(g, 3, initial_state=st, final_state=st)
    assert torch.equal(o3, o1)
    assert torch.equal(st, s1)


def test_blocked_bf16_output():
    x, g = _inputs(2, 36 * 64, 2, 128, seed=44)
    o1, s1 = _call(g, 1, o_dtype=torch.bfloat16)
    o4, s4 = _call(g, 4, o_dtype=torch.bfloat16)
    assert torch.equal(o4, o1)
    assert torch.equal(s4, s1)


def _call_coop(g, **kw):
    """Default schedule: one cooperative launch (prep CTAs publish records,
    scan CTAs consume them) whenever the scan grid leaves 32 SMs free."""
    out = kda.kda_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], g["initial_state"], **kw)
    torch.cuda.synchronize()
    kda.kda_check()
    return out


@pytest.mark.parametrize("B,T,H,d", [(2, 33 * 64 + 37, 3, 128), (1, 64, 1, 128), (3, 20 * 64 + 1, 5, 64),
                                     (2, 4096, 16, 128)])
def test_cooperative_schedule_bit_identical(B, T, H, d):
    x, g = _inputs(B, T, H, d, seed=70 + H)
    o1, s1 = _call(g, 1)
    o2, s2 = _call_coop(g)
    assert torch.equal(o2, o1)
    assert torch.equal(s2, s1)
    o3, s3 = _call_coop(g, output_final_state=False, o_dtype=torch.bfloat16)
    o4, _ = _call(g, 1, output_final_state=False, o_dtype=torch.bfloat16)
    assert s3 is None and torch.equal(o3, o4)


@pytest.mark.parametrize("d,H", [(128, 32), (64, 64)])
def test_persistent_scan_matches_one_cta_per_item(d, H):
    """A dense batch of more than four scan items per SM (B = 10: 640 items of
    64 value columns) runs prep then scan, with one
    persistent scan CTA per SM taking every gridDim.x-th item: each sequence's
    results are bit-identical to the same sequence alone (a one-launch
    schedule with one scan CTA per item); one pair of heads is checked
    against the oracle."""
    x, g = _inputs(10, 130, H, d, seed=910)
    o, sT = _call(g, 0)
    for b in (0, 3, 9):
        one = {k: (None if v is None else v[b:b + 1].contiguous()) for k, v in g.items()}
        o1, s1 = _call(one, 0)
        assert torch.equal(o[b:b + 1], o1) and torch.equal(sT[b:b + 1], s1)
    b, hs = 9, [0, H - 1]
    flat = lambda t: f64(t[b, :, hs])
    o_ref, s_ref = oracle.recurrence(flat(x["q"]), flat(x["k"]), flat(x["v"]), f64(x["beta"][b, :, hs]),
                                     flat(x["log_alpha"]), np.array([0, 130]), f64(x["initial_state"][b:b + 1, hs]))
    assert norm_max_err(f64(o[b, :, hs]), o_ref) <= TOL_BF16
    assert norm_max_err(f64(sT[b:b + 1, hs]), s_ref) <= TOL_BF16
