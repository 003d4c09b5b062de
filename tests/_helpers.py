"""Shared test helpers: tensor conversion and the parity metric."""
import numpy as np
import torch


def f64(t):
    """Exact fp64 copy of a tensor's values (bf16 values are upcast exactly)."""
    if t is None:
        return None
    return t.detach().to("cpu", torch.float64).numpy()


def norm_max_err(got, ref):
    """max |got - ref| / RMS(ref): the parity metric of the layer's tolerances."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    rms = np.sqrt(np.mean(ref * ref))
    return float(np.max(np.abs(got - ref)) / max(rms, 1e-300))


TOL_F32 = 1e-4   # fp32 q/k/v, fp32 state
TOL_BF16 = 2e-2  # bf16 q/k/v, fp32 state
