#!/usr/bin/env python
"""Benchmark of the KDA layer on B200.

One step = one chunkwise forward (gate cumsum, intra-chunk A, UT transform,
state scan, intra-chunk output, final state) over the long-context workload
(B=1, H=32, T=131072, d_k=d_v=128, bf16 q/k/v, fp32 state, chunk 64; the
largest single-GPU configuration), inputs resident in HBM (5.4 GB, far larger
than the 126 MB L2).  The prefill (B=2, H=16, T=4096) and packed variable-length
(8 sequences, 65536 tokens, H=32) forwards, the layer variants and the decode
step (256 sequences x 32 heads, 64 consecutive tokens) are timed in the same
run and reported under "other_workloads" and "decode".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: one process per GPU (torchrun); every rank runs its own copy of the
workload with its own seed (weak scaling, no data-path collective); the time is
the max over ranks.  --impl reference times the fp64 CPU oracle on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA chunk-fwd tokens/s & TFLOP/s (% roofline); decode-step state GB/s on 1 B200"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- work model
def bytes_per_token_head(dk, dv, elem, o_elem=2):
    """Algorithmic HBM bytes per (token, head): q, k, v in (elem bytes each),
    o out (o_elem bytes), log alpha (fp32 per key channel) and beta (fp32) in.
    With bf16 q/k/v/o and d = 128 this is the 1540 B of the roofline; the
    library's default fp32 o adds 2 d_v bytes (1796 B)."""
    return elem * (2 * dk + dv) + o_elem * dv + 4 * dk + 4


def flops_per_token_head(dk, dv, C=64):
    """Algorithmic FLOPs per (token, head) of the chunk forward, triangles at
    half: A and P ((C-1) and (C+1) pairs of d_k), U-like 2C d_v, the four
    state products 6 d_k d_v, the UT transform C^2/3."""
    return (2 * (C - 1) + (C + 1)) * dk + 2 * C * dv + 6 * dk * dv + C * C / 3.0


def bwd_flops_per_token_head(dk, dv, C=64):
    """Algorithmic FLOPs per (token, head) of the chunkwise backward (dense
    products, per chunk, divided by C): the forward recompute (MA and P over
    d_k, X = Kh S, U = T Y, the state update, the UT transform) and the adjoint
    products (dU, dY, dP, dT, T^T dT T^T, the three d_k-wide gradient
    accumulations and the state-gradient update)."""
    fwd = 2 * (2 * C * C * dk) + 2 * C * dk * dv + 2 * C * C * dv + 2 * dk * C * dv + C ** 3 / 3
    adj = (2 * C * C * dv + 2 * C * dk * dv          # dU = P^T dO + Kl dS'
           + 2 * C * C * dv + 2 * C * C * dv         # dY = T^T dU, dP = dO U^T
           + 2 * C * C * dv + 2 * 2 * C * C * C      # dT = dU Y^T, T^T dT T^T
           + 3 * 2 * C * dk * dv + 5 * 2 * C * C * dk  # dO S^T, dX S^T, U dS'^T; dP, dMA products
           + 2 * 2 * dk * C * dv)                    # dS = Qh^T dO + Kh^T dX
    return (fwd + adj) / C


def dplr_flops_per_token_head(dk, dv, C=64):
    """Algorithmic FLOPs per (token, head) of the diagonal-plus-low-rank chunk
    forward (dense products per chunk / C): the four intra-chunk products over
    d_k, (e^Gx a) S and A_ak V, U = T W, the output's three products, the two
    state-update products, and the triangular solve."""
    per_chunk = (4 * 2 * C * C * dk + 2 * C * dk * dv + 2 * C * C * dv + 2 * C * C * dv
                 + 2 * C * dk * dv + 2 * 2 * C * C * dv + 2 * 2 * dk * C * dv + C ** 3 / 3)
    return per_chunk / C


def fp32_alu_peak_tflops(device=None):
    """CUDA-core fp32 peak from unit counts: SMs x 128 FP32 lanes x 2 FLOP (FMA)
    x the maximum SM clock (1965 MHz on these B200s)."""
    nsm = torch.cuda.get_device_properties(device).multi_processor_count if device is not None else 148
    return nsm * 128 * 2 * 1.965e9 / 1e12


def chunk_work(B, T, H, dk, dv, elem=2, o_elem=2, state_in=True, state_out=True):
    th = B * T * H
    nbytes = th * bytes_per_token_head(dk, dv, elem, o_elem)
    nbytes += (int(state_in) + int(state_out)) * B * H * dk * dv * 4
    return nbytes, th * flops_per_token_head(dk, dv)


def decode_state_bytes(N, H, dk, dv):
    return 2 * N * H * dk * dv * 4


# ----------------------------------------------------------------------------- distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return world, rank, local


def init_dist(world, backend):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def reduce_max(x: float, world: int, device) -> float:
    """Max of a per-rank scalar over all ranks (the timing rule)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world, device=None):
    if world > 1:
        if device is not None and device.type == "cuda":
            torch.distributed.barrier(device_ids=[device.index])
        else:
            torch.distributed.barrier()


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms in the background."""
    FIELDS = ("index,timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()
        return False

    def summary(self):
        rows = [r for r in csv.reader(io.StringIO(getattr(self, "out", ""))) if len(r) >= 10]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[2]) for r in rows if num(r[2]) is not None]
        mx = [num(r[3]) for r in rows if num(r[3]) is not None]
        power = [num(r[4]) for r in rows if num(r[4]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].strip().lower() == "active"})
        # "under load": samples at or above the median power draw
        load = sm
        if power and len(power) == len(sm):
            cut = statistics.median(power)
            load = [s for s, p in zip(sm, power) if p >= cut] or sm
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- helpers
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {k: p[k] for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = {
    # the files whose code a recorded ncu capture of each path depends on
    "chunk_fwd_prefill": ["kda_chunk_split.cu", "kda_tc_util.cuh", "kda_sm100.cuh", "kda_common.cuh"],
    "chunk_fwd_long": ["kda_chunk_split.cu", "kda_tc_util.cuh", "kda_sm100.cuh", "kda_common.cuh"],
    "decode_step": ["kda_decode.cu", "kda_common.cuh"],
}


def kernel_source_hash(kernel_key="chunk_fwd_prefill"):
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_delta_rule_133_b200", "csrc")
    for name in KERNEL_SOURCES[kernel_key]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_key):
    """Per-launch DRAM bytes of a kernel from a committed ncu summary, or None
    when the kernel sources changed since that capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel_key)
    if not rec or rec.get("source_hash") != kernel_source_hash(kernel_key):
        return None
    return rec.get("dram_bytes_per_launch")


def chunk_launches(B, T, H, dv, device, varlen=False):
    """Kernels one chunk-forward call launches (the library's rule): dense
    inputs whose scan grid (B * H * dv / 64 CTAs) leaves at least 32 SMs run as
    one cooperative kernel (prep and scan CTAs together); otherwise a prep and
    a scan kernel, plus the index kernel of a packed batch."""
    nsm = torch.cuda.get_device_properties(device).multi_processor_count
    if not varlen and B * H * (dv // 64) + 32 <= nsm:
        return 1
    return 3 if varlen else 2


def event_pairs(n):
    return [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]


def chunk_roofline(nbytes, nbytes_f32o, nflops, launch_s, traffic=None):
    """Roofline of one chunk-forward call: algorithmic bytes (bf16 o: 1540 B
    per token-head plus the states) over the call's CUDA-event time, against the measured copy
    bandwidth; the fp32-o byte count (what the default call writes) beside it."""
    pk, kind = peaks()
    achieved = nbytes / launch_s / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / pk["hbm_gbs"], "traffic": traffic, "peak_kind": f"{kind} copy bandwidth",
            "bytes_per_launch": nbytes, "launch_ms": launch_s * 1e3,
            "fp32_o": {"bytes_per_launch": nbytes_f32o, "achieved": nbytes_f32o / launch_s / 1e9,
                       "frac": nbytes_f32o / launch_s / 1e9 / pk["hbm_gbs"]},
            "tensor_frac": nflops / launch_s / 1e12 / pk["bf16_tflops"]}


def dense_work(w, state_in):
    nbytes, nflops = chunk_work(w.B, w.T, w.H, w.dk, w.dv, state_in=state_in)
    nbytes_f32o, _ = chunk_work(w.B, w.T, w.H, w.dk, w.dv, o_elem=4, state_in=state_in)
    return nbytes, nbytes_f32o, nflops


# ----------------------------------------------------------------------------- our arm
def run_ours(args, world, rank, local):
    import gated_delta_rule_133_b200 as kda
    from gated_delta_rule_133_b200.inputs import WORKLOADS, make_inputs

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    init_dist(world, "nccl")
    w = WORKLOADS["long"]
    stream = torch.cuda.current_stream(device)

    d = make_inputs(w, device, seed=w.seed + 1000 * rank)
    o = torch.empty(w.B, w.T, w.H, w.dv, dtype=torch.float32, device=device)
    sN = torch.empty(w.B, w.H, w.dk, w.dv, dtype=torch.float32, device=device)
    ws = torch.empty(kda.chunk_fwd_workspace_size(w.B, w.T, w.H, w.dk, w.dv), dtype=torch.uint8, device=device)
    nbytes, nbytes_f32o, nflops = dense_work(w, state_in=d["initial_state"] is not None)
    set_bytes = sum(t.numel() * t.element_size() for t in d.values() if t is not None)

    def step(i):
        kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["log_alpha"], d["initial_state"],
                          o=o, final_state=sN, workspace=ws, stream=stream)

    sampler = ClockSampler(device.index)
    with sampler:
        for i in range(args.warmup):
            step(i)
        torch.cuda.synchronize(device)
        kda.kda_check()
        ev = event_pairs(args.steps)
        barrier(world, device)
        torch.cuda.synchronize(device)
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step(i)
            ev[i][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(device)
        barrier(world, device)
        kda.kda_check()
        elapsed = reduce_max(t_start.elapsed_time(t_end) / 1e3, world, device)
        launch_s = statistics.mean(a.elapsed_time(b) for a, b in ev) / 1e3

        # ---- end to end through the public API from pinned host buffers
        host = {k: (None if v is None else v.cpu()) for k, v in d.items()}
        del d, o, sN
        torch.cuda.empty_cache()
        e2e = run_e2e(kda, host, w, device, stream, world, ws, steps=max(3, min(args.steps, 10)))
        del host, ws
        torch.cuda.empty_cache()

        # ---- decode: 64 consecutive steps over 256 x 32 fp32 states
        dec = run_decode(kda, device, stream, world, rank, max(3, args.warmup))

        # ---- the other chunk-forward workloads (context)
        others = {} if args.skip_others else run_other_workloads(kda, device, stream, world, rank,
                                                                 reps=max(3, min(args.steps, 20)))

    clocks = sampler.summary()
    tokens = w.B * w.T * world
    value = tokens * args.steps / elapsed
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"long context: B={w.B} H={w.H} T={w.T} d_k={w.dk} d_v={w.dv} chunk={w.chunk}, "
                               "bf16 q/k/v, fp32 state and fp32 output, log alpha = -softplus(z), z ~ N(-1, 1), "
                               "zero initial state",
                   "global_batch": w.B * world, "seq_len": w.T, "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2: one input set of {set_bytes / 1e9:.1f} GB"},
        "tflops": nflops * world * args.steps / elapsed / 1e12,
        "roofline": chunk_roofline(nbytes, nbytes_f32o, nflops, launch_s, recorded_traffic("chunk_fwd_long")),
        "decode": dec,
        "other_workloads": others,
        "e2e": e2e,
        "gpu_launches": args.steps * chunk_launches(w.B, w.T, w.H, w.dv, device),
        "clocks": clocks,
    }
    return line, rank


def run_decode(kda, device, stream, world, rank, warmup):
    from gated_delta_rule_133_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS["decode"]
    x = make_inputs(w, device, seed=w.seed + 1000 * rank)
    state = x["initial_state"].clone()
    o = torch.empty(w.B, w.H, w.dv, dtype=torch.float32, device=device)

    def one(s):
        kda.kda_recurrent_step(x["q"][s], x["k"][s], x["v"][s], x["beta"][s], x["log_alpha"][s], state,
                               o=o, stream=stream)

    for s in range(warmup):
        one(s % w.T)
    torch.cuda.synchronize(device)
    state.copy_(x["initial_state"])
    ev = event_pairs(w.T)
    barrier(world, device)
    torch.cuda.synchronize(device)
    for s in range(w.T):
        ev[s][0].record(stream)
        one(s)
        ev[s][1].record(stream)
    torch.cuda.synchronize(device)
    per = [a.elapsed_time(b) / 1e3 for a, b in ev]
    total = reduce_max(ev[0][0].elapsed_time(ev[-1][1]) / 1e3, world, device)
    nbytes = decode_state_bytes(w.B, w.H, w.dk, w.dv)
    pk, kind = peaks()
    gbs = nbytes * world * w.T / total / 1e9
    per_launch = nbytes / statistics.mean(per) / 1e9
    return {"workload": f"decode: {w.B} sequences x H={w.H}, d_k=d_v={w.dk}, fp32 state "
                        f"({w.B * w.H * w.dk * w.dv * 4 / 2**20:.0f} MiB), {w.T} consecutive steps",
            "value": gbs, "unit": "GB/s (state read + write)", "us_per_step": total / w.T * 1e6,
            "roofline": {"bound": "hbm", "achieved": per_launch, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": per_launch / pk["hbm_gbs"], "traffic": recorded_traffic("decode_step"),
                         "peak_kind": f"{kind} copy bandwidth"},
            "gpu_launches": w.T}


def run_other_workloads(kda, device, stream, world, rank, reps=20):
    """The prefill (B2 H16 T4096) and varlen (8 packed sequences, 65536 tokens,
    H32) chunk forwards, the same 65536 tokens packed as 1024 short sequences
    (lengths 16..112), and the prefill shape with the two layer variants (one
    gate per head; no erase term): one warm-up launch, `reps` timed launches
    each, inputs resident in HBM."""
    from gated_delta_rule_133_b200.inputs import WORKLOADS, make_inputs
    out = {}
    for name in ("prefill", "varlen", "varlen_1024", "prefill_head_gate", "prefill_no_erase"):
        w = WORKLOADS[name.split("_")[0]]
        if name == "varlen_1024":
            w = type(w)(**{**w.__dict__, "B": 1024, "extra": {"min_len": 16, "max_len": 112}})
        d = make_inputs(w, device, seed=w.seed + 1000 * rank)
        desc = f"{name}: {w.B * w.T if w.kind != 'varlen' else w.T} tokens, H={w.H}, d_k=d_v={w.dk}, bf16 q/k/v, fp32 o and state"
        if w.kind == "varlen":
            desc += f", {w.B} sequences of {w.extra['min_len']}..{w.extra['max_len']} tokens"
        kw = {}
        gate_bytes = 4 * w.dk
        if name.startswith("prefill"):
            if name == "prefill_head_gate":
                d["log_alpha"] = d["log_alpha"][..., 0].contiguous()
                kw["head_gate"] = True
                gate_bytes = 4
                desc += ", one forget gate per (token, head)"
            if name == "prefill_no_erase":
                kw["erase"] = False
                desc += ", no erase term"
            o = torch.empty(w.B, w.T, w.H, w.dv, dtype=torch.float32, device=device)
            sN = torch.empty(w.B, w.H, w.dk, w.dv, dtype=torch.float32, device=device)
            mode = (1 if kw.get("head_gate") else 0) | (0 if kw.get("erase", True) else 2)
            ws = torch.empty(kda.chunk_fwd_workspace_size(w.B, w.T, w.H, w.dk, w.dv, mode=mode), dtype=torch.uint8,
                             device=device)
            call = lambda: kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["log_alpha"], d["initial_state"],
                                             o=o, final_state=sN, stream=stream, workspace=ws, **kw)
            tokens, s_in, s_out = w.B * w.T, w.B, w.B
            launches = chunk_launches(w.B, w.T, w.H, w.dv, device)
        else:
            cu = d["cu_seqlens"]
            nseq = cu.numel() - 1
            o = torch.empty(w.T, w.H, w.dv, dtype=torch.float32, device=device)
            sN = torch.empty(nseq, w.H, w.dk, w.dv, dtype=torch.float32, device=device)
            ws = torch.empty(kda.varlen_fwd_workspace_size(nseq, w.T, w.H, w.dk, w.dv), dtype=torch.uint8,
                             device=device)
            call = lambda: kda.kda_varlen_fwd(d["q"], d["k"], d["v"], d["beta"], d["log_alpha"], cu, None,
                                              o=o, final_state=sN, stream=stream, workspace=ws)
            tokens, s_in, s_out = w.T, 0, nseq
            launches = chunk_launches(1, w.T, w.H, w.dv, device, varlen=True)
        call()
        torch.cuda.synchronize(device)
        ev = event_pairs(reps)
        barrier(world, device)
        for a, b in ev:
            a.record(stream)
            call()
            b.record(stream)
        torch.cuda.synchronize(device)
        kda.kda_check()
        t = reduce_max(statistics.mean(a.elapsed_time(b) for a, b in ev) / 1e3, world, device)
        per_th = lambda o_elem: bytes_per_token_head(w.dk, w.dv, 2, o_elem) - 4 * w.dk + gate_bytes
        states = (s_in + s_out) * w.H * w.dk * w.dv * 4
        nbytes = tokens * w.H * per_th(2) + states
        nbytes_f32o = tokens * w.H * per_th(4) + states
        nflops = tokens * w.H * flops_per_token_head(w.dk, w.dv)
        out[name] = {"workload": desc, "ms": t * 1e3, "tokens_per_s": tokens * world / t,
                     "roofline": chunk_roofline(nbytes, nbytes_f32o, nflops, t,
                                                recorded_traffic("chunk_fwd_prefill") if name == "prefill" else None),
                     "gpu_launches_per_call": launches}
        if not name.startswith("prefill_"):   # the layer's FLOPs (the variants do less arithmetic)
            out[name]["tflops"] = nflops * world / t / 1e12
        del d, o, sN, ws
        torch.cuda.empty_cache()
    out["prefill_backward"] = run_backward(kda, device, stream, world, rank, reps=max(3, min(reps, 5)))
    out["prefill_dplr"] = run_dplr(kda, device, stream, world, rank, reps=max(3, min(reps, 5)))
    return out


def run_dplr(kda, device, stream, world, rank, reps=3):
    """The diagonal-plus-low-rank transition's chunk forward (fp32, CUDA cores)
    on the prefill shape, with a, b ~ N(0, 0.7^2 / d_k)."""
    from gated_delta_rule_133_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS["prefill"]
    d = make_inputs(w, device, seed=w.seed + 1000 * rank)
    g = torch.Generator(device=device).manual_seed(11 + rank)
    ab = [(torch.randn(w.B, w.T, w.H, w.dk, generator=g, device=device) * 0.7 / w.dk ** 0.5).to(torch.bfloat16)
          for _ in range(2)]
    o = torch.empty(w.B, w.T, w.H, w.dv, device=device)
    sN = torch.empty(w.B, w.H, w.dk, w.dv, device=device)
    ws = torch.empty(kda.dplr_fwd_workspace_size(w.B, w.T, w.H, w.dk, w.dv), dtype=torch.uint8, device=device)
    call = lambda: kda.kda_dplr_fwd(d["q"], d["k"], d["v"], ab[0], ab[1], d["log_alpha"], d["initial_state"],
                                    o=o, final_state=sN, stream=stream, workspace=ws)
    call()
    torch.cuda.synchronize(device)
    ev = event_pairs(reps)
    barrier(world, device)
    for a, b in ev:
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize(device)
    kda.kda_check()
    t = reduce_max(statistics.mean(a.elapsed_time(b) for a, b in ev) / 1e3, world, device)
    nflops = w.B * w.T * w.H * dplr_flops_per_token_head(w.dk, w.dv)
    peak = fp32_alu_peak_tflops(device)
    return {"workload": f"diagonal-plus-low-rank transition, prefill shape: B={w.B} H={w.H} T={w.T} "
                        f"d_k=d_v={w.dk}, bf16 q/k/v/a/b, fp32 o and state, CUDA-core kernel",
            "ms": t * 1e3, "tokens_per_s": w.B * w.T * world / t,
            "roofline": {"bound": "alu", "achieved": nflops / t / 1e12, "peak": peak, "unit": "TFLOP/s",
                         "frac": nflops / t / 1e12 / peak, "peak_kind": "fp32 FMA: SMs x 128 lanes x 2 x 1965 MHz",
                         "flops_per_launch": nflops},
            "gpu_launches_per_call": 1}


def run_backward(kda, device, stream, world, rank, reps=3):
    """The chunkwise backward (fp32, CUDA cores) on the prefill shape: gradients
    of sum(o * dO) + sum(S_T * dS_T) for random dO, dS_T."""
    from gated_delta_rule_133_b200.inputs import WORKLOADS, make_inputs
    w = WORKLOADS["prefill"]
    d = make_inputs(w, device, seed=w.seed + 1000 * rank)
    g = torch.Generator(device=device).manual_seed(7 + rank)
    do = torch.randn(w.B, w.T, w.H, w.dv, generator=g, device=device)
    dsT = torch.randn(w.B, w.H, w.dk, w.dv, generator=g, device=device)
    call = lambda: kda.kda_chunk_bwd(d["q"], d["k"], d["v"], d["beta"], d["log_alpha"], d["initial_state"], do, dsT,
                                     stream=stream)
    call()
    torch.cuda.synchronize(device)
    ev = event_pairs(reps)
    barrier(world, device)
    for a, b in ev:
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize(device)
    kda.kda_check()
    t = reduce_max(statistics.mean(a.elapsed_time(b) for a, b in ev) / 1e3, world, device)
    th = w.B * w.T * w.H
    nflops = th * bwd_flops_per_token_head(w.dk, w.dv)
    peak = fp32_alu_peak_tflops(device)
    achieved = nflops / t / 1e12
    return {"workload": f"backward, prefill shape: B={w.B} H={w.H} T={w.T} d_k=d_v={w.dk}, bf16 q/k/v, fp32 "
                        "gradients, CUDA-core kernel",
            "ms": t * 1e3, "tokens_per_s": w.B * w.T * world / t,
            "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "peak_kind": "fp32 FMA: SMs x 128 lanes x 2 x 1965 MHz",
                         "flops_per_launch": nflops},
            "gpu_launches_per_call": 1}


def run_e2e(kda, host_inputs, w, device, stream, world, ws, steps):
    """Same metric through the public API with pinned host buffers, as a
    pipelined loop over steps: every step copies its inputs host->device on a
    copy-in stream, runs the chunk forward on the compute stream and reads o
    and the final state back on a copy-out stream; two buffer sets let step
    i + 1's inputs travel while step i computes and its results return (PCIe
    is full duplex).  Events order each buffer set's reuse."""
    host = {k: (None if v is None else v.pin_memory()) for k, v in host_inputs.items()}
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    sets = []
    for _ in range(2):
        dev = {k: (None if v is None else torch.empty_like(v, device=device)) for k, v in host.items()}
        o_d = torch.empty(w.B, w.T, w.H, w.dv, dtype=torch.float32, device=device)
        s_d = torch.empty(w.B, w.H, w.dk, w.dv, dtype=torch.float32, device=device)
        o_h = torch.empty(w.B, w.T, w.H, w.dv, dtype=torch.float32).pin_memory()
        s_h = torch.empty(w.B, w.H, w.dk, w.dv, dtype=torch.float32).pin_memory()
        sets.append((dev, o_d, s_d, o_h, s_h))
    d2h = sets[0][3].numel() * 4 + sets[0][4].numel() * 4
    s_in = torch.cuda.Stream(device)
    s_out = torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()
    done_compute = [None, None]   # compute of the set's previous step (inputs free)
    done_out = [None, None]       # copy-out of the set's previous step (outputs free)

    def one(i):
        j = i % 2
        dev, o_d, s_d, o_h, s_h = sets[j]
        with torch.cuda.stream(s_in):
            if done_compute[j] is not None:
                s_in.wait_event(done_compute[j])
            for k, v in host.items():
                if v is not None:
                    dev[k].copy_(v, non_blocking=True)
            e_in = ev()
            e_in.record(s_in)
        stream.wait_event(e_in)
        if done_out[j] is not None:
            stream.wait_event(done_out[j])
        kda.kda_chunk_fwd(dev["q"], dev["k"], dev["v"], dev["beta"], dev["log_alpha"], dev["initial_state"],
                          o=o_d, final_state=s_d, workspace=ws, stream=stream)
        e_c = ev()
        e_c.record(stream)
        done_compute[j] = e_c
        with torch.cuda.stream(s_out):
            s_out.wait_event(e_c)
            o_h.copy_(o_d, non_blocking=True)
            s_h.copy_(s_d, non_blocking=True)
            e_o = ev()
            e_o.record(s_out)
        done_out[j] = e_o

    for i in range(2):
        one(i)
    torch.cuda.synchronize(device)
    barrier(world, device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    s_in.wait_stream(stream)
    for i in range(steps):
        one(i)
    stream.wait_stream(s_out)
    b.record(stream)
    torch.cuda.synchronize(device)
    t = reduce_max(a.elapsed_time(b) / 1e3, world, device)
    return {"value": w.B * w.T * world * steps / t, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "pipelined": "2 buffer sets, copy-in / compute / copy-out streams"}


# ----------------------------------------------------------------------------- oracle arm
ORACLE_SAMPLE_TOKENS = 65536


def oracle_sample(heads_max=16):
    """Times the fp64 oracle on a bounded sample of the long-context workload:
    every head (in groups of up to `heads_max`, one thread per head, at most
    the host's cores) of one sequence of ORACLE_SAMPLE_TOKENS tokens drawn with
    the workload's recipe, each group drawn with its own seed.  The recurrence
    costs the same per token, so the rate scales to the whole workload (131072
    tokens x 32 heads).  Returns its tokens/s, the threads used and the sample
    description."""
    import numpy as np
    import oracle
    from gated_delta_rule_133_b200.inputs import WORKLOADS, draw_tokens
    w = WORKLOADS["long"]
    cores = os.cpu_count() or 1
    heads = max(1, min(heads_max, w.H, cores))
    groups = max(1, min(w.H // heads, 2))
    T = ORACLE_SAMPLE_TOKENS
    f = lambda x: x.to(torch.float64).numpy()
    dt = 0.0
    for g in range(groups):
        d = draw_tokens(T, heads, w.dk, w.dv, w.dtype, w.gate_mu, w.seed + g, "cpu")
        args = [f(d[n]) for n in ("q", "k", "v", "beta", "log_alpha")]
        del d
        t0 = time.perf_counter()
        oracle.recurrence(*args, np.array([0, T]), None, nthreads=heads)
        dt += time.perf_counter() - t0
        del args
    full_time = dt * (w.T / T) * (w.H / (heads * groups))
    return {"value": w.B * w.T / full_time, "unit": "tokens/s", "cores": heads, "kind": "oracle",
            "sample": f"long-context recipe, {groups} x {heads} heads x {T} tokens ({dt:.1f} s, {heads} threads), "
                      f"scaled to {w.H} heads x {w.T} tokens"}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    vals = []
    info = None
    for i in range(args.warmup + args.steps):
        info = oracle_sample()
        if i >= args.warmup:
            vals.append(info["value"])
    value = statistics.mean(vals) if vals else info["value"]
    from gated_delta_rule_133_b200.inputs import WORKLOADS
    w = WORKLOADS["long"]
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": w.B * w.T / value * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"long context: B={w.B} H={w.H} T={w.T} d_k={w.dk} d_v={w.dv} chunk={w.chunk}, "
                                   "bf16 q/k/v, fp32 state and fp32 output, log alpha = -softplus(z), z ~ N(-1, 1), "
                                   "zero initial state",
                       "global_batch": w.B * world, "seq_len": w.T, "parallelism": f"replicas x{world}",
                       "oracle": "fp64 CPU token recurrence"},
            "cpu_baseline": {**info, "value": value},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_case(args):
    """One library call of the named workload, --warmup + --steps times on cuda:0
    (for profiler command lines: a handful of launches, nothing else timed)."""
    import gated_delta_rule_133_b200 as kda
    from gated_delta_rule_133_b200.inputs import WORKLOADS, make_inputs
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    name = {"backward": "prefill", "dplr": "prefill"}.get(args.case, args.case)
    w = WORKLOADS[name]
    if args.case == "long" and args.case_tokens:
        w = type(w)(**{**w.__dict__, "T": args.case_tokens})
    d = make_inputs(w, device)
    if args.case == "decode":
        state = d["initial_state"].clone()
        call = lambda i: kda.kda_recurrent_step(d["q"][i % w.T], d["k"][i % w.T], d["v"][i % w.T], d["beta"][i % w.T],
                                                d["log_alpha"][i % w.T], state)
    elif args.case == "backward":
        g = torch.Generator(device=device).manual_seed(7)
        do = torch.randn(w.B, w.T, w.H, w.dv, generator=g, device=device)
        call = lambda i: kda.kda_chunk_bwd(d["q"], d["k"], d["v"], d["beta"], d["log_alpha"], d["initial_state"], do)
    elif args.case == "dplr":
        g = torch.Generator(device=device).manual_seed(11)
        a, b = [(torch.randn(w.B, w.T, w.H, w.dk, generator=g, device=device) * 0.7 / w.dk ** 0.5).to(torch.bfloat16)
                for _ in range(2)]
        call = lambda i: kda.kda_dplr_fwd(d["q"], d["k"], d["v"], a, b, d["log_alpha"], d["initial_state"])
    else:
        ws = torch.empty(kda.chunk_fwd_workspace_size(w.B, w.T, w.H, w.dk, w.dv), dtype=torch.uint8, device=device)
        call = lambda i: kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["log_alpha"], d["initial_state"],
                                           workspace=ws)
    for i in range(args.warmup + args.steps):
        call(i)
    torch.cuda.synchronize(device)
    kda.kda_check()


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--skip-others", action="store_true", help="skip the prefill / varlen / variant timings")
    ap.add_argument("--case", choices=["prefill", "long", "decode", "backward", "dplr"], default=None,
                    help="profiling aid: run only this call --steps times after --warmup calls, print nothing")
    ap.add_argument("--case-tokens", type=int, default=0,
                    help="with --case long: tokens of the sequence (default: the workload's 131072)")
    args = ap.parse_args(argv)
    world, rank, local = dist_env()
    if args.case:
        run_case(args)
        return 0
    if args.impl == "reference":
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    line, rank = run_ours(args, world, rank, local)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_sample()
    elif rank == 0:
        line["cpu_baseline"] = None
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
