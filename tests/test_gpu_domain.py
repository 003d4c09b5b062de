"""GPU: gates at and past the edge of the chunk kernels' numerical domain.

The tensor-core chunk forward, the backward and the DPLR forward factor the
decay inside a 64-token chunk around its middle row, with the factors clamped
at exp(+-80).  A chunk whose gates decay a channel by more than 80 nats
between its first or last row and the middle is outside their domain: the
kernels then flag the chunk, kda_check() reports KDA_WARN_DOMAIN, and the
results stay finite but lose accuracy.  Inside the domain nothing is reported
and the usual bars hold.  The CUDA-core chunk forward splits the decay by
16-row blocks with every factor at most 1, and the decode step needs no
factors: neither has a limit.

Gates here are a constant log alpha = -s on every channel, so the decay from
the first row to the middle row (31 tokens) is 31 s nats.
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


def _inputs(s, dtype, T=192, H=2, d=128, seed=700):
    w = Workload("domain", "dense", 1, T, H, d, d, dtype, -3.0, 0.05, seed=seed)
    x = make_inputs(w, "cpu")
    x["log_alpha"] = torch.full_like(x["log_alpha"], -s)
    return x


def _oracle(x):
    B, T, H = x["q"].shape[:3]
    flat = lambda t: f64(t).reshape(B * T, H, *t.shape[3:])
    return oracle.recurrence(flat(x["q"]), flat(x["k"]), flat(x["v"]), f64(x["beta"]).reshape(B * T, H),
                             flat(x["log_alpha"]), np.array([0, T]), f64(x["initial_state"]))


def _run_fwd(x, cuda_cores=False):
    g = {n: (None if t is None else t.to(DEV)) for n, t in x.items()}
    o, sT = kda.kda_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], g["initial_state"],
                              cuda_cores=cuda_cores)
    torch.cuda.synchronize()
    return o, sT


@pytest.mark.parametrize("dtype,tol", [("bf16", TOL_BF16), ("fp32", 1e-4)])
def test_inside_the_domain_nothing_is_reported(dtype, tol):
    x = _inputs(2.5, dtype)          # 31 x 2.5 = 77.5 nats: inside
    o, sT = _run_fwd(x)
    kda.kda_check()
    o_ref, s_ref = _oracle(x)
    assert norm_max_err(f64(o).reshape(o_ref.shape), o_ref) <= tol
    assert norm_max_err(f64(sT), s_ref) <= tol


@pytest.mark.parametrize("s", [2.7, 4.0, 8.0])
def test_past_the_domain_is_reported_and_finite(s):
    """Tensor-core path, 31 s > 80 nats: KDA_WARN_DOMAIN, finite outputs; the
    error against the oracle is recorded in the assertion message of the
    finiteness check."""
    x = _inputs(s, "bf16")
    o, sT = _run_fwd(x)
    with pytest.raises(kda.KdaError) as e:
        kda.kda_check()
    assert e.value.status == kda._lib.KDA_WARN_DOMAIN
    kda.kda_check()   # the status word was cleared
    o_ref, s_ref = _oracle(x)
    err = norm_max_err(f64(o).reshape(o_ref.shape), o_ref)
    assert torch.isfinite(o).all() and torch.isfinite(sT).all(), f"s = {s}: error {err:.3e}"


@pytest.mark.parametrize("dtype,tol", [("fp32", 1e-4), ("bf16", 1e-4)])
@pytest.mark.parametrize("s", [2.7, 8.0, 30.0])
def test_cuda_core_path_has_no_domain_limit(dtype, tol, s):
    """The 16-row segmentation of the CUDA-core kernel keeps every factor at
    most 1: gates far past the tensor-core path's edge are as exact as weak
    ones, with nothing reported (bf16 inputs through KDA_MODE_CUDA_CORES are
    computed in fp32 too)."""
    x = _inputs(s, dtype, T=200)
    o, sT = _run_fwd(x, cuda_cores=True)
    kda.kda_check()
    o_ref, s_ref = _oracle(x)
    assert norm_max_err(f64(o).reshape(o_ref.shape), o_ref) <= tol
    assert norm_max_err(f64(sT), s_ref) <= tol


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_cuda_core_path_mixed_chunks(dtype):
    """One sequence whose odd chunks decay 8 nats per token and whose even
    chunks carry the recipe's gates: the CUDA-core kernel takes the middle-row
    split for some chunks and the 16-row segmentation for the others, with one
    state carried across; both stay within the fp32 bar."""
    w = Workload("domain", "dense", 1, 300, 2, 128, 128, dtype, -3.0, 0.05, seed=702)
    x = make_inputs(w, "cpu")
    strong = (torch.arange(300) // 64) % 2 == 1
    x["log_alpha"][:, strong] = -8.0
    o, sT = _run_fwd(x, cuda_cores=True)
    kda.kda_check()
    o_ref, s_ref = _oracle(x)
    assert norm_max_err(f64(o).reshape(o_ref.shape), o_ref) <= 1e-4
    assert norm_max_err(f64(sT), s_ref) <= 1e-4


def test_backward_and_dplr_report_the_domain_too():
    """The backward and the DPLR forward factor their chunks the same way and
    flag the same chunks (the DPLR outputs stay finite)."""
    x = _inputs(4.0, "bf16", T=128)
    g = {n: (None if t is None else t.to(DEV)) for n, t in x.items()}
    do = torch.randn_like(g["v"], dtype=torch.float32)
    grads = kda.kda_chunk_bwd(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], g["initial_state"], do)
    torch.cuda.synchronize()
    with pytest.raises(kda.KdaError) as e:
        kda.kda_check()
    assert e.value.status == kda._lib.KDA_WARN_DOMAIN
    a = (0.05 * torch.randn_like(g["k"], dtype=torch.float32)).to(torch.bfloat16)
    o, sT = kda.kda_dplr_fwd(g["q"], g["k"], g["v"], a, a, g["log_alpha"], g["initial_state"])
    torch.cuda.synchronize()
    with pytest.raises(kda.KdaError) as e:
        kda.kda_check()
    assert e.value.status == kda._lib.KDA_WARN_DOMAIN
    assert torch.isfinite(o).all() and torch.isfinite(sT).all()


def test_decode_has_no_domain_limit():
    """The token recurrence needs no factorisation: strong gates are exact."""
    from gated_delta_rule_133_b200.inputs import WORKLOADS
    w = Workload("dec", "decode", 4, 1, 2, 128, 128, "bf16", -3.0, 0.02, seed=701)
    x = make_inputs(w, "cpu")
    la = torch.full_like(x["log_alpha"][0], -8.0)
    state = x["initial_state"].to(DEV).clone()
    o = kda.kda_recurrent_step(*(x[n][0].to(DEV) for n in ("q", "k", "v", "beta")), la.to(DEV), state)
    torch.cuda.synchronize()
    kda.kda_check()
    o_ref, s_ref = oracle.recurrent_step(*(f64(x[n][0]) for n in ("q", "k", "v", "beta")), f64(la),
                                         f64(x["initial_state"]))
    assert norm_max_err(f64(o), o_ref) <= TOL_BF16
