"""GPU: kda_chunk_fwd_noalloc, the forward with every intermediate in the
library's fixed per-device area (collected last: it leaves that area in use).

It must give results bit-identical to kda_chunk_fwd (same kernels; only the
location of the operand records and of the carried state differs), over a
ring of blocks small enough that records of a block are overwritten two
blocks later, and it must not allocate device memory."""
import pytest
import torch

import gated_delta_rule_133_b200 as kda
from gated_delta_rule_133_b200 import _lib
from gated_delta_rule_133_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _inputs(B, T, H, d, seed):
    w = Workload("noalloc", "dense", B, T, H, d, d, "bf16", -3.0, 0.05, seed=seed)
    return {k: (None if v is None else v.to(DEV)) for k, v in make_inputs(w, "cpu").items()}


def _both(g, **kw):
    args = (g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], g["initial_state"])
    ref = kda.kda_chunk_fwd(*args, **kw)
    out = kda.kda_chunk_fwd_noalloc(*args, **kw)
    torch.cuda.synchronize()
    kda.kda_check()
    return ref, out


@pytest.mark.parametrize("B,T,H,d", [
    (2, 4096 + 37, 4, 128),     # one block
    (4, 640 + 17, 64, 128),     # 256 (sequence, head) pairs: 2 chunks per block, ring reused
    (4, 640, 64, 64),
])
def test_noalloc_matches_chunk_fwd(B, T, H, d):
    g = _inputs(B, T, H, d, seed=50 + H)
    (o1, s1), (o2, s2) = _both(g)
    assert torch.equal(o2, o1)
    assert torch.equal(s2, s1)


def test_noalloc_without_final_state_and_bf16_output():
    """Carried state in the area (1 chunk per block with 256 pairs)."""
    g = _inputs(4, 640 + 5, 64, 128, seed=61)
    (o1, _), (o2, s2) = _both(g, output_final_state=False, o_dtype=torch.bfloat16)
    assert s2 is None
    assert torch.equal(o2, o1)


def test_noalloc_in_place_state():
    g = _inputs(2, 1024 + 9, 8, 128, seed=62)
    o1, s1 = kda.kda_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], g["initial_state"])
    st = g["initial_state"].clone()
    o2, _ = kda.kda_chunk_fwd_noalloc(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], st, final_state=st)
    torch.cuda.synchronize()
    assert torch.equal(o2, o1)
    assert torch.equal(st, s1)


def test_noalloc_in_place_state_across_ring_blocks():
    """256 (sequence, head) pairs, 11 chunks: 2 chunks per block, 6 blocks, each
    block reading and writing the caller's state in place."""
    g = _inputs(4, 657, 64, 128, seed=65)
    o1, s1 = kda.kda_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], g["initial_state"])
    st = g["initial_state"].clone()
    o2, _ = kda.kda_chunk_fwd_noalloc(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], st, final_state=st)
    torch.cuda.synchronize()
    kda.kda_check()
    assert torch.equal(o2, o1)
    assert torch.equal(st, s1)


def test_noalloc_single_block_needs_no_second_slot():
    """1000 (sequence, head) pairs of one chunk, no final state: the records of
    one block fill most of the area, which is enough when there is one block."""
    g = _inputs(10, 50, 100, 128, seed=66)
    (o1, _), (o2, s2) = _both(g, output_final_state=False)
    assert s2 is None
    assert torch.equal(o2, o1)


def test_noalloc_rejects_oversize():
    g = _inputs(20, 64, 64, 128, seed=63)
    with pytest.raises(_lib.KdaError) as e:
        kda.kda_chunk_fwd_noalloc(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], g["initial_state"])
    assert e.value.status == _lib.KDA_ERR_UNSUPPORTED


def test_noalloc_allocates_nothing():
    """Device free memory is unchanged across calls (after a first call has
    loaded the module and its area)."""
    g = _inputs(4, 640 + 17, 64, 128, seed=64)
    o = torch.empty(4, 640 + 17, 64, 128, device=DEV)
    s = torch.empty(4, 64, 128, 128, device=DEV)
    args = (g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], g["initial_state"])
    kda.kda_chunk_fwd_noalloc(*args, o=o, final_state=s)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        kda.kda_chunk_fwd_noalloc(*args, o=o, final_state=s)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
