"""Device-side failure detection without a GPU fault.

Every spin wait in the library's kernels is bounded (about one second of
globaltimer) and, when it gives up, records SWITCH_ERR_DEVICE_TIMEOUT in the
workspace status word instead of trapping.  The self-test kernel waits on an
mbarrier that nothing completes, with that same bounded wait: the test checks
that the wait ends, that switch_check reports the timeout once, and that the
CUDA context still runs a layer correctly afterwards.
"""
import time

import numpy as np
import pytest
import torch

import sparse_mixture_experts_fp32_b200 as sm
from sparse_mixture_experts_fp32_b200 import synth

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    t0 = time.time()
    sm.selftest_wait_timeout(ws)
    assert sm.switch_check(ws) == 8  # SWITCH_ERR_DEVICE_TIMEOUT
    elapsed = time.time() - t0
    assert 0.5 < elapsed < 30, elapsed
    assert sm.switch_check(ws) == 0  # reading the status clears it
    # the context is still healthy: a small layer runs and reports no error
    wl = synth.WORKLOADS["base8"]
    inp = synth.inputs(wl, T=256)
    dev = {k: (torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).cuda() if v is not None and v.dtype == np.uint16
               else (torch.from_numpy(v).cuda() if v is not None else None)) for k, v in inp.items()}
    out = sm.layer_fwd(dev["x"], dev["w_r"], dev["w_in"], dev["w_out"], capacity_factor=1.25)
    assert sm.switch_check(out["workspace"]) == 0
    assert int(out["counts"].sum().item()) == 256
