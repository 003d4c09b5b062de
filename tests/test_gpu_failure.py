"""Failure detection on the GPU without any fault: a bounded device-side wait
that nothing satisfies runs out, the kernel records KDA_ERR_TIMEOUT and exits,
the host reads it through kda_check(), and the context stays usable."""
import pytest
import torch

import gated_delta_rule_133_b200 as kda
from gated_delta_rule_133_b200 import _lib
from gated_delta_rule_133_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu


def _stream():
    return torch.cuda.current_stream().cuda_stream


def test_bounded_wait_runs_out_and_is_reported():
    lib = _lib.load()
    torch.cuda.synchronize()
    assert lib.kda_check(_stream()) == _lib.KDA_OK
    assert lib.kda_selftest_timeout(1 << 20, _stream()) == _lib.KDA_OK   # ~0.5 ms budget
    assert lib.kda_check(_stream()) == _lib.KDA_ERR_TIMEOUT
    assert lib.kda_check(_stream()) == _lib.KDA_OK                       # read and cleared
    with pytest.raises(kda.KdaError) as e:
        lib.kda_selftest_timeout(1 << 16, _stream())
        kda.kda_check()
    assert e.value.status == _lib.KDA_ERR_TIMEOUT


def test_context_usable_after_timeout():
    lib = _lib.load()
    lib.kda_selftest_timeout(1 << 16, _stream())
    assert lib.kda_check(_stream()) == _lib.KDA_ERR_TIMEOUT
    w = Workload("after", "dense", 1, 100, 2, 128, 128, "bf16", -3.0, 0.02, seed=3)
    x = {k: (None if v is None else v.cuda()) for k, v in make_inputs(w, "cpu").items()}
    o, s = kda.kda_chunk_fwd(x["q"], x["k"], x["v"], x["beta"], x["log_alpha"], x["initial_state"])
    torch.cuda.synchronize()
    kda.kda_check()
    assert torch.isfinite(o).all() and torch.isfinite(s).all()
