"""Router statistics (switch_router_stats) on the CUDA path against the oracle: the mean entropy
of the router probabilities, the dropped fraction, the capacity utilisation and the busiest
expert's load, for every router kernel (staged, tiled, tensor-core) and for top-2 routing."""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_fp32_b200 as sm
from sparse_mixture_experts_fp32_b200 import synth
from parity import to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def orc():
    return oracle.Oracle()


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return sm.lib()


CASES = [("tiny_fp32", 64, 0), ("base8", 3000, 0), ("base128_skew", 5000, 0), ("large128", 2000, 0),
         ("base128_skew", 3000, sm.SWITCH_FLAG_SIMT_ROUTER), ("bigexpert64", 700, 0)]


@pytest.mark.parametrize("name,T,flags", CASES, ids=[f"{c[0]}-{c[2]}" for c in CASES])
@pytest.mark.parametrize("top2", [False, True], ids=["top1", "top2"])
def test_router_stats(orc, name, T, flags, top2):
    wl = synth.WORKLOADS[name]
    x, w_r, bias = synth.activations(wl, T=T), synth.router_weight(wl), synth.router_bias(wl)
    C = sm.switch_capacity(T, wl.num_experts, wl.capacity_factor)
    f = flags | sm.SWITCH_FLAG_ROUTER_STATS
    route = sm.route_top2 if top2 else sm.route
    r = route(to_device(x), to_device(w_r), capacity=C, logit_bias=to_device(bias), d_ff=wl.d_ff, flags=f)
    assert sm.switch_check(r["workspace"]) == 0
    st = sm.router_stats(r, T, wl.d_model, wl.d_ff, to_device(x).dtype).cpu().numpy().astype(np.float64)
    o = orc.route(x, w_r, bias, capacity=C, want_probs=True)
    ref = orc.router_stats(o["probs"], r["counts"].cpu().numpy(), C)  # counts: the GPU's (top-2: assignments)
    assert abs(st[0] - ref["entropy"]) <= 1e-5 * ref["entropy"], (st[0], ref["entropy"])
    assert abs(st[1] - ref["drop_fraction"]) <= 1e-6 * max(ref["drop_fraction"], 1e-30) + 1e-7
    assert abs(st[2] - ref["capacity_utilisation"]) <= 1e-6 * ref["capacity_utilisation"]
    assert abs(st[3] - ref["max_load"]) <= 1e-6 * ref["max_load"]


def test_router_stats_without_the_flag_gives_no_entropy():
    wl = synth.WORKLOADS["base8"]
    T = 1000
    x = to_device(synth.activations(wl, T=T))
    r = sm.route(x, to_device(synth.router_weight(wl)), capacity_factor=1.25, d_ff=wl.d_ff)
    r["flags"] = 0
    st = sm.router_stats(r, T, wl.d_model, wl.d_ff, x.dtype).cpu().numpy()
    assert np.isnan(st[0]) and np.all(np.isfinite(st[1:]))
