"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Metric: max |gpu - oracle| / RMS(oracle), separately for o and for the final
state.  Bars: 1e-4 for fp32 q/k/v, 2e-2 for bf16 q/k/v (fp32 state).  The
oracle sees exactly the values the GPU sees (bf16 inputs upcast exactly).
"""
import numpy as np
import pytest
import torch

import oracle
import gated_delta_rule_133_b200 as kda
from gated_delta_rule_133_b200.inputs import WORKLOADS, Workload, draw_tokens, make_inputs, cu_from_lengths
from tests._helpers import TOL_BF16, TOL_F32, f64, norm_max_err

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _dense_oracle(d, B, T):
    """Oracle on dense [B, T, H, ...] inputs."""
    H = d["q"].shape[2]
    flat = lambda x: f64(x).reshape(B * T, H, *x.shape[3:])
    cu = np.arange(B + 1, dtype=np.int64) * T
    return oracle.recurrence(flat(d["q"]), flat(d["k"]), flat(d["v"]), f64(d["beta"]).reshape(B * T, H),
                             flat(d["log_alpha"]), cu, f64(d["initial_state"]))


def _to(d, dev):
    return {k: (None if v is None else v.to(dev)) for k, v in d.items()}


def _run_dense(w, **override):
    d = make_inputs(w, "cpu", **override)
    B, T = d["q"].shape[:2]
    g = _to(d, DEV)
    o, sT = kda.kda_chunk_fwd(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], g["initial_state"])
    torch.cuda.synchronize()
    kda.kda_check()
    o_ref, s_ref = _dense_oracle(d, B, T)
    H, dv = o.shape[2], o.shape[3]
    return f64(o).reshape(B * T, H, dv), f64(sT), o_ref, s_ref


def test_tiny_fp32_config():
    """Tiny workload: B1 H2 T256 d64 fp32, zero initial state."""
    o, sT, o_ref, s_ref = _run_dense(WORKLOADS["tiny"])
    assert norm_max_err(o, o_ref) <= TOL_F32
    assert norm_max_err(sT, s_ref) <= TOL_F32


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
@pytest.mark.parametrize("d,dtype", [(128, "bf16"), (64, "bf16"), (128, "fp32")])
def test_chunk_fwd_ragged(T, d, dtype):
    w = Workload("case", "dense", 2, T, 3, d, d, dtype, -3.0, 0.05, seed=10 + T)
    o, sT, o_ref, s_ref = _run_dense(w)
    tol = TOL_F32 if dtype == "fp32" else TOL_BF16
    assert norm_max_err(o, o_ref) <= tol
    assert norm_max_err(sT, s_ref) <= tol


def test_chunk_fwd_mixed_head_dims():
    w = Workload("case", "dense", 1, 130, 2, 128, 64, "bf16", -1.0, 0.05, seed=21)
    o, sT, o_ref, s_ref = _run_dense(w)
    assert norm_max_err(o, o_ref) <= TOL_BF16
    assert norm_max_err(sT, s_ref) <= TOL_BF16


def test_strong_forgetting_gates():
    """z ~ N(-1, 1): in-chunk relative decays span ~e^-26 (long-context gates)."""
    w = Workload("case", "dense", 1, 512, 4, 128, 128, "bf16", -1.0, 0.0, seed=22)
    o, sT, o_ref, s_ref = _run_dense(w)
    assert norm_max_err(o, o_ref) <= TOL_BF16
    assert norm_max_err(sT, s_ref) <= TOL_BF16


def test_zero_tokens_passes_state_through():
    H, d = 2, 128
    s0 = torch.randn(3, H, d, d, device=DEV)
    e = torch.empty(3, 0, H, d, device=DEV, dtype=torch.bfloat16)
    o, sT = kda.kda_chunk_fwd(e, e, e, torch.empty(3, 0, H, device=DEV),
                              torch.empty(3, 0, H, d, device=DEV), s0)
    torch.cuda.synchronize()
    assert torch.equal(sT, s0)


def test_split_resume_equals_one_pass():
    w = Workload("case", "dense", 1, 300, 2, 128, 128, "bf16", -3.0, 0.02, seed=23)
    d = _to(make_inputs(w, "cpu"), DEV)
    o, sT = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["log_alpha"], d["initial_state"])
    cut = 100  # not a chunk multiple
    sl = lambda x, a, b: x[:, a:b].contiguous()
    o1, s1 = kda.kda_chunk_fwd(*(sl(d[n], 0, cut) for n in ("q", "k", "v", "beta", "log_alpha")),
                               d["initial_state"])
    o2, s2 = kda.kda_chunk_fwd(*(sl(d[n], cut, 300) for n in ("q", "k", "v", "beta", "log_alpha")), s1)
    torch.cuda.synchronize()
    o12 = torch.cat([o1, o2], dim=1)
    assert norm_max_err(f64(o12), f64(o)) <= TOL_BF16
    assert norm_max_err(f64(s2), f64(sT)) <= TOL_BF16


def test_in_place_final_state():
    w = Workload("case", "dense", 2, 130, 2, 128, 128, "bf16", -3.0, 0.02, seed=24)
    d = _to(make_inputs(w, "cpu"), DEV)
    o_a, s_a = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["log_alpha"], d["initial_state"])
    s = d["initial_state"].clone()
    o_b, s_b = kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["log_alpha"], s, final_state=s)
    torch.cuda.synchronize()
    assert torch.equal(o_a, o_b) and torch.equal(s_a, s)


def _varlen_case(lens, H, d, dtype, seed, s0_std=0.05):
    cu = cu_from_lengths(lens)
    t = draw_tokens(int(cu[-1]), H, d, d, dtype, -3.0, seed, "cpu", init_states=len(lens), init_std=s0_std)
    t["cu_seqlens"] = torch.from_numpy(cu)
    return t


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_varlen_small(dtype):
    lens = [1, 63, 64, 65, 0, 200, 129]
    d = _varlen_case(lens, 2, 128, dtype, 31)
    g = _to(d, DEV)
    o, sN = kda.kda_varlen_fwd(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], g["cu_seqlens"],
                               g["initial_state"])
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.recurrence(f64(d["q"]), f64(d["k"]), f64(d["v"]), f64(d["beta"]),
                                     f64(d["log_alpha"]), d["cu_seqlens"].numpy(), f64(d["initial_state"]))
    tol = TOL_F32 if dtype == "fp32" else TOL_BF16
    assert norm_max_err(f64(o), o_ref) <= tol
    assert norm_max_err(f64(sN), s_ref) <= tol
    # the empty sequence passes its initial state through unchanged
    assert torch.equal(sN[4], g["initial_state"][4])
    # packed equals per-sequence dense calls
    cu = d["cu_seqlens"].numpy()
    for n in (1, 5):
        a, b = cu[n], cu[n + 1]
        on, sn = kda.kda_chunk_fwd(*(g[x][a:b].unsqueeze(0).contiguous() for x in ("q", "k", "v", "beta", "log_alpha")),
                                   g["initial_state"][n:n + 1].contiguous())
        torch.cuda.synchronize()
        assert norm_max_err(f64(on[0]), f64(o[a:b])) <= tol
        assert norm_max_err(f64(sn[0]), f64(sN[n])) <= tol


@pytest.mark.parametrize("d,dtype", [(128, "bf16"), (64, "fp32"), (128, "fp32")])
def test_recurrent_step_matches_oracle(d, dtype):
    N, H, steps = 5, 3, 8
    w = Workload("dec", "decode", N, steps, H, d, d, dtype, -3.0, 0.02, seed=41)
    x = make_inputs(w, "cpu")
    state = x["initial_state"].to(DEV).clone()
    S_ref = f64(x["initial_state"])
    tol = TOL_F32 if dtype == "fp32" else TOL_BF16
    for s in range(steps):
        g = {n: x[n][s].to(DEV) for n in ("q", "k", "v", "beta", "log_alpha")}
        o = kda.kda_recurrent_step(g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], state)
        torch.cuda.synchronize()
        o_ref, S_ref = oracle.recurrent_step(*(f64(x[n][s]) for n in ("q", "k", "v", "beta", "log_alpha")), S_ref)
        assert norm_max_err(f64(o), o_ref) <= tol
        assert norm_max_err(f64(state), S_ref) <= tol


def test_decode_steps_equal_chunk_forward():
    """Repeated single-token steps give the chunk forward's result (same math)."""
    N, H, d, steps = 3, 2, 128, 70
    w = Workload("dec", "decode", N, steps, H, d, d, "fp32", -3.0, 0.02, seed=42)
    x = _to(make_inputs(w, "cpu"), DEV)
    state = x["initial_state"].clone()
    outs = []
    for s in range(steps):
        outs.append(kda.kda_recurrent_step(x["q"][s], x["k"][s], x["v"][s], x["beta"][s], x["log_alpha"][s], state))
    o_dec = torch.stack(outs, 1)                               # [N, steps, H, d]
    tr = lambda t: t.transpose(0, 1).contiguous()            # [steps, N, ...] -> [N, steps, ...]
    o_chk, s_chk = kda.kda_chunk_fwd(tr(x["q"]), tr(x["k"]), tr(x["v"]), tr(x["beta"]), tr(x["log_alpha"]),
                                     x["initial_state"])
    torch.cuda.synchronize()
    assert norm_max_err(f64(o_dec), f64(o_chk)) <= 1e-4
    assert norm_max_err(f64(state), f64(s_chk)) <= 1e-4


def test_bf16_output_is_the_rounded_fp32_output():
    """o_dtype=bf16 stores exactly the fp32 result rounded to nearest even."""
    w = Workload("case", "dense", 2, 150, 3, 128, 128, "bf16", -3.0, 0.02, seed=25)
    d = _to(make_inputs(w, "cpu"), DEV)
    args = (d["q"], d["k"], d["v"], d["beta"], d["log_alpha"], d["initial_state"])
    o32, s32 = kda.kda_chunk_fwd(*args)
    o16, s16 = kda.kda_chunk_fwd(*args, o_dtype=torch.bfloat16)
    lens = [70, 0, 130]
    v = _to(_varlen_case(lens, 2, 128, "bf16", 26), DEV)
    vargs = (v["q"], v["k"], v["v"], v["beta"], v["log_alpha"], v["cu_seqlens"], v["initial_state"])
    vo32, _ = kda.kda_varlen_fwd(*vargs)
    vo16, _ = kda.kda_varlen_fwd(*vargs, o_dtype=torch.bfloat16)
    x = _to(make_inputs(Workload("dec", "decode", 4, 1, 2, 128, 128, "bf16", -3.0, 0.02, seed=27), "cpu"), DEV)
    st_a, st_b = x["initial_state"].clone(), x["initial_state"].clone()
    dargs = tuple(x[n][0] for n in ("q", "k", "v", "beta", "log_alpha"))
    do32 = kda.kda_recurrent_step(*dargs, st_a)
    do16 = kda.kda_recurrent_step(*dargs, st_b, o_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert o16.dtype == torch.bfloat16 and torch.equal(o16, o32.to(torch.bfloat16))
    assert torch.equal(s16, s32)
    assert torch.equal(vo16, vo32.to(torch.bfloat16))
    assert torch.equal(do16, do32.to(torch.bfloat16)) and torch.equal(st_a, st_b)


@pytest.mark.parametrize("d", [128, 64])
def test_tensor_core_and_cuda_core_kernels_agree(d):
    """bf16 inputs go to the tcgen05 kernel; KDA_MODE_CUDA_CORES sends them to
    the CUDA-core kernel.  Both meet the bar against the oracle."""
    w = Workload("case", "dense", 2, 333, 2, d, d, "bf16", -1.0, 0.05, seed=28)
    d_cpu = make_inputs(w, "cpu")
    g = _to(d_cpu, DEV)
    args = (g["q"], g["k"], g["v"], g["beta"], g["log_alpha"], g["initial_state"])
    o_tc, s_tc = kda.kda_chunk_fwd(*args)
    o_cc, s_cc = kda.kda_chunk_fwd(*args, cuda_cores=True)
    torch.cuda.synchronize()
    o_ref, s_ref = _dense_oracle(d_cpu, 2, 333)
    flat = lambda t: f64(t).reshape(2 * 333, 2, d)
    assert norm_max_err(flat(o_tc), o_ref) <= TOL_BF16
    assert norm_max_err(flat(o_cc), o_ref) <= 1e-4
    assert norm_max_err(f64(s_tc), s_ref) <= TOL_BF16
    assert norm_max_err(f64(s_cc), s_ref) <= 1e-4
