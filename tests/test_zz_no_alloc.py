"""switch_route_noalloc, the routing call that allocates nothing, checked
against switch_route.

Some users of this library cannot allocate device memory at the point where
they route tokens: they run under a host framework that owns every device
allocation and forbids new ones while it executes, or in a process that
reserved all of its device memory up front.  switch_route_noalloc keeps its
scratch in a static array inside the library instead of a caller-supplied
workspace.  Here it is called through the C ABI several times in a row, on
different problems (so that anything one call leaves in the shared array would
show in the next), and each result is compared with switch_route's on the same
inputs: ids, slots, counts and slot_token bit for bit, gates and aux within the
parity tolerances.  The pairs cover both ways the capacity scan runs (inside the
slot assignment for small histograms, and as its own kernel, which adds to and
then resets a ticket kept in the shared array), the all-float32 path and an
empty group.  The test also checks that a call leaves the device's free memory
unchanged, that a group too large for the static array is refused before
anything runs, and that switch_check_noalloc reads (and clears) the status word
kept in the static array: OK after a routing call, SWITCH_ERR_DEVICE_TIMEOUT
after the bounded-wait self-test.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import sparse_mixture_experts_fp32_b200 as sm
from sparse_mixture_experts_fp32_b200 import synth

pytestmark = pytest.mark.gpu

AUX_RTOL = 1e-5   # the tolerance the parity tests use for the aux loss
GATE_ATOL = 1e-5  # ... and for the gates


def _dev(a):
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _outputs(T, N, C):
    return dict(expert=torch.full((T,), -7, dtype=torch.int32, device="cuda"),
                gate=torch.full((T,), -7.0, dtype=torch.float32, device="cuda"),
                slot=torch.full((T,), -7, dtype=torch.int32, device="cuda"),
                counts=torch.full((N,), -7, dtype=torch.int32, device="cuda"),
                slot_token=torch.full((N * C,), -7, dtype=torch.int32, device="cuda"),
                aux=torch.full((1,), -7.0, dtype=torch.float32, device="cuda"))


def _call_noalloc(d, x, w_r, bias, out):
    L = sm.lib()
    p = lambda t: None if t is None else t.data_ptr()
    stream = torch.cuda.current_stream().cuda_stream
    return L.switch_route_noalloc(ctypes.byref(d), p(x), p(w_r), p(bias), p(out["expert"]), p(out["gate"]),
                                  p(out["slot"]), p(out["counts"]), p(out["slot_token"]), p(out["aux"]), stream)


def _compare(name, T, flags=0):
    wl = synth.WORKLOADS[name]
    x = _dev(synth.activations(wl, T=T))
    w_r = _dev(synth.router_weight(wl))
    bias = _dev(synth.router_bias(wl))
    N = wl.num_experts
    C = sm.switch_capacity(T, N, wl.capacity_factor)
    ref = sm.route(x, w_r, capacity=C, logit_bias=bias, d_ff=wl.d_ff, flags=flags)  # with a workspace
    assert sm.switch_check(ref["workspace"]) == 0
    d = sm.dims(T, wl.d_model, wl.d_ff, N, C, x.dtype, flags)
    out = _outputs(T, N, C)
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    status = _call_noalloc(d, x, w_r, bias, out)
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    assert status == 0, sm.STATUS.get(status, status)
    for k in ("expert", "slot", "counts", "slot_token"):
        assert torch.equal(out[k], ref[k]), k
    if T > 0:
        assert torch.max(torch.abs(out["gate"] - ref["gate"])).item() <= GATE_ATOL
        assert abs(out["aux"].item() - ref["aux"].item()) <= AUX_RTOL * abs(ref["aux"].item())
    else:
        assert out["aux"].item() == 0.0
    return free_before, free_after


def test_noalloc_route_matches_route_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    # first call: 128 experts, skewed routing, many drops
    _compare("base128_skew", 5000)
    # second call right after it, different N, T and tile count
    free_before, free_after = _compare("base8", 3000)
    assert free_after == free_before, "switch_route_noalloc changed the device's free memory"


def test_noalloc_route_with_the_scan_kernel_twice_in_a_row():
    """The separate scan kernel adds to a ticket in the shared array and resets it;
    two calls back to back show whether the second starts from a clean ticket."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    flags = sm.SWITCH_FLAG_SEPARATE_SCAN
    _compare("base128_skew", 5000, flags)
    _compare("large128", 4000, flags)
    free_before, free_after = _compare("base8", 3000, flags)
    assert free_after == free_before


def test_noalloc_route_float32_and_empty_group():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _compare("tiny_fp32", 64)   # all-float32 router
    _compare("base8", 0)        # no tokens: counts 0, aux 0, every slot empty
    _compare("tiny_fp32", 64)   # and a normal call again after the empty one


def test_noalloc_route_refuses_groups_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    T, N, C = 1 << 20, 256, 4096  # needs ~50 MB of scratch, far above 4 MiB
    small = torch.zeros(64, dtype=torch.float32, device="cuda")
    d = sm.dims(T, 64, 64, N, C, sm.SWITCH_BF16)
    out = _outputs(16, N, 1)
    status = _call_noalloc(d, small, small, None, out)
    assert status == 9  # SWITCH_ERR_TOO_LARGE
    torch.cuda.synchronize()
    assert torch.all(out["counts"] == -7) and torch.all(out["aux"] == -7.0)


def test_noalloc_status_word_is_readable():
    """switch_check_noalloc: OK after a routing call; after the bounded-wait self-test (one block that
    gives up waiting on an mbarrier nothing completes, after about a second, and exits normally) it
    reports SWITCH_ERR_DEVICE_TIMEOUT once, clears the word, and routing still matches switch_route."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _compare("base8", 1000)
    assert sm.switch_check_noalloc() == 0
    sm.selftest_wait_timeout_noalloc()
    assert sm.switch_check_noalloc() == 8  # SWITCH_ERR_DEVICE_TIMEOUT
    assert sm.switch_check_noalloc() == 0  # read and cleared
    _compare("base8", 1000)
    assert sm.switch_check_noalloc() == 0

