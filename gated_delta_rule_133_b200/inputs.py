"""Seeded synthetic inputs for the KDA layer.

This module only draws random numbers with the stated distributions and lays
them out; it holds none of the layer's arithmetic.  The tests hand the same
tensors to the CUDA path and to the CPU oracle.

Distributions (the workloads' own recipe): q, k ~ N(0, 1) then L2-normalised
over d_k per (token, head); v ~ N(0, 1); beta = sigmoid(N(0, 1)); per-channel
log alpha = -softplus(z) with z ~ N(mu, 1) (mu = -3, or -1 for the
strong-forgetting long-context case); initial state zeros or N(0, 0.02^2).
Draw order inside one generator: q, k, v, beta logits, z, initial state.
Everything is drawn in fp32, then q, k, v are cast to the requested dtype;
beta, log alpha and states stay fp32.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

_DT = {"fp32": torch.float32, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "dense", "varlen" or "decode"
    B: int                    # batch (dense), sequence count (varlen, decode)
    T: int                    # tokens per sequence (dense), total tokens (varlen), steps (decode)
    H: int
    dk: int
    dv: int
    dtype: str                # dtype of q, k, v, o
    gate_mu: float            # mean of z in log alpha = -softplus(z)
    init_std: float           # 0 -> zero initial state
    chunk: int = 64
    seed: int = 0
    extra: dict = field(default_factory=dict, compare=False, hash=False)


# The five synthetic workloads the layer is measured and checked on.
WORKLOADS = {
    "tiny": Workload("tiny", "dense", 1, 256, 2, 64, 64, "fp32", -3.0, 0.0, seed=0),
    "prefill": Workload("prefill", "dense", 2, 4096, 16, 128, 128, "bf16", -3.0, 0.02, seed=1),
    "varlen": Workload("varlen", "varlen", 8, 65536, 32, 128, 128, "bf16", -3.0, 0.0, seed=2,
                       extra={"min_len": 512, "max_len": 16384}),
    "long": Workload("long", "dense", 1, 131072, 32, 128, 128, "bf16", -1.0, 0.0, seed=3),
    "decode": Workload("decode", "decode", 256, 64, 32, 128, 128, "bf16", -3.0, 0.02, seed=4),
}


def varlen_lengths(n: int, total: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """n lengths drawn uniformly in [lo, hi], rescaled to sum to `total`
    (rounded; the rounding remainder goes onto the last length); the draw is
    repeated until every length lies in [lo, hi]."""
    rng = np.random.default_rng(seed)
    for _ in range(1000):
        u = rng.integers(lo, hi, size=n, endpoint=True).astype(np.float64)
        lens = np.round(u * (total / u.sum())).astype(np.int64)
        lens[-1] += total - lens.sum()
        if lens.min() >= lo and lens.max() <= hi:
            return lens
    raise RuntimeError("could not draw admissible lengths")


def cu_from_lengths(lens) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(np.asarray(lens, dtype=np.int64))]).astype(np.int32)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def draw_tokens(T: int, H: int, dk: int, dv: int, dtype: str, gate_mu: float,
                seed: int, device="cpu", init_states: int = 0, init_std: float = 0.0):
    """Token-major packed tensors: q, k [T, H, dk]; v [T, H, dv]; beta [T, H];
    log_alpha [T, H, dk]; initial_state [init_states, H, dk, dv] or None."""
    g = _gen(device, seed)
    q = torch.randn(T, H, dk, generator=g, device=device)
    q = q / q.norm(dim=-1, keepdim=True).clamp_min(1e-30)
    k = torch.randn(T, H, dk, generator=g, device=device)
    k = k / k.norm(dim=-1, keepdim=True).clamp_min(1e-30)
    v = torch.randn(T, H, dv, generator=g, device=device)
    beta = torch.sigmoid(torch.randn(T, H, generator=g, device=device))
    z = torch.randn(T, H, dk, generator=g, device=device) + gate_mu
    log_alpha = -torch.nn.functional.softplus(z)
    s0 = None
    if init_states and init_std > 0:
        s0 = torch.randn(init_states, H, dk, dv, generator=g, device=device) * init_std
    t = _DT[dtype]
    return {"q": q.to(t).contiguous(), "k": k.to(t).contiguous(), "v": v.to(t).contiguous(),
            "beta": beta.contiguous(), "log_alpha": log_alpha.contiguous(),
            "initial_state": None if s0 is None else s0.contiguous()}


def make_inputs(w: Workload, device="cpu", **override):
    """Inputs of one workload (fields may be overridden, e.g. a shorter T for
    tests).  Dense: tensors carry a leading batch dim [B, T, ...].  Varlen: a
    single packed batch with ``cu_seqlens`` (int32).  Decode: ``steps`` sets of
    per-token inputs [steps, N, H, ...] plus the starting state."""
    if override:
        w = Workload(**{**w.__dict__, **override})
    if w.kind == "dense":
        d = draw_tokens(w.B * w.T, w.H, w.dk, w.dv, w.dtype, w.gate_mu, w.seed, device,
                        init_states=w.B, init_std=w.init_std)
        for name in ("q", "k", "v", "beta", "log_alpha"):
            d[name] = d[name].reshape(w.B, w.T, *d[name].shape[1:])
        return d
    if w.kind == "varlen":
        lens = w.extra.get("lengths")
        if lens is None:
            lens = varlen_lengths(w.B, w.T, w.extra["min_len"], w.extra["max_len"], w.seed)
        cu = cu_from_lengths(lens)
        d = draw_tokens(int(cu[-1]), w.H, w.dk, w.dv, w.dtype, w.gate_mu, w.seed, device,
                        init_states=w.B, init_std=w.init_std)
        d["cu_seqlens"] = torch.from_numpy(cu).to(device)
        return d
    if w.kind == "decode":
        N, steps = w.B, w.T
        d = draw_tokens(steps * N, w.H, w.dk, w.dv, w.dtype, w.gate_mu, w.seed, device,
                        init_states=N, init_std=w.init_std)
        for name in ("q", "k", "v", "beta", "log_alpha"):
            d[name] = d[name].reshape(steps, N, *d[name].shape[1:])
        if d["initial_state"] is None:
            d["initial_state"] = torch.zeros(N, w.H, w.dk, w.dv, device=device)
        return d
    raise ValueError(w.kind)
