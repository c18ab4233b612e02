"""Backward pass of the layer on the CUDA path (through the C ABI) against the
fp64 backward oracle, element by element.

The loss is L = sum(y * dy) + g_aux * aux with a seeded upstream gradient dy.
The expert GEMMs run on tensor cores with bfloat16 operands and float32
accumulation, so each gradient tensor is compared with the bf16 bar of the
forward outputs: max-abs error <= 2e-2 x RMS of the oracle's tensor.  Routing
is the GPU forward's own (the oracle recomputes it; near-tie tokens, whose
expert can differ, are excluded from these cases by construction of the
check: the GPU ids must equal the oracle's on every token).
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_fp32_b200 as sm
from sparse_mixture_experts_fp32_b200 import synth
from parity import to_device

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module")
def orc():
    return oracle.Oracle()


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return sm.lib()


def _compare(name, got, ref, report):
    got = got.double().cpu().numpy() if isinstance(got, torch.Tensor) else got
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = float(np.abs(got - ref).max())
    report[name] = err / rms if rms > 0 else err
    if rms == 0.0:
        assert err == 0.0, f"{name}: expected exact zeros, max |got| = {err}"
    else:
        assert err <= TOL * rms, f"{name}: max-abs error {err:.3e} > {TOL} x RMS {rms:.3e}"


def run_backward(orc, inp, C, g_aux, seed, check_bias=True):
    T, d = inp["x"].shape
    rng = np.random.default_rng(seed)
    dy = rng.standard_normal((T, d)).astype(np.float32)
    dev = {k: to_device(v) for k, v in inp.items()}
    fwd = sm.layer_fwd(dev["x"], dev["w_r"], dev["w_in"], dev["w_out"], capacity=C, logit_bias=dev["bias"],
                       flags=sm.SWITCH_FLAG_TRAINING)
    g = sm.layer_bwd(fwd, dev["x"], dev["w_r"], dev["w_in"], dev["w_out"], torch.from_numpy(dy).cuda(), g_aux,
                     logit_bias=dev["bias"])
    assert sm.switch_check(fwd["workspace"]) == 0
    o = orc.route(inp["x"], inp["w_r"], inp["bias"], capacity=C)
    assert np.array_equal(fwd["expert"].cpu().numpy(), o["expert"]), "routing differs (near tie in a gradient case)"
    ref = orc.layer_bwd(inp["x"], inp["w_r"], inp["w_in"], inp["w_out"], dy.astype(np.float64), g_aux,
                        bias=inp["bias"], capacity=C)
    rep = {}
    _compare("dx", g["dx"], ref["dx"], rep)
    _compare("dw_r", g["dw_r"], ref["dw_r"], rep)
    if check_bias and inp["bias"] is not None:
        _compare("dbias", g["dbias"], ref["dbias"], rep)
    kept = np.minimum(o["counts"], C) > 0
    _compare("dw_in", g["dw_in"][torch.from_numpy(kept).cuda()], ref["dw_in"][kept], rep)
    _compare("dw_out", g["dw_out"][torch.from_numpy(kept).cuda()], ref["dw_out"][kept], rep)
    # experts without kept tokens get exactly zero weight gradients
    if (~kept).any():
        idle = torch.from_numpy(~kept).cuda()
        assert torch.all(g["dw_in"][idle] == 0) and torch.all(g["dw_out"][idle] == 0)
    # a dropped token's gradient is the router part only: zero when g_aux = 0 and dy only reaches kept tokens
    return rep, fwd, g


SMALL = [("base8", 600), ("base128_skew", 3000), ("large128", 900), ("bigexpert64", 200)]


@pytest.mark.parametrize("name,T", SMALL, ids=[n for n, _ in SMALL])
def test_backward_small(orc, name, T, record_property):
    wl = synth.WORKLOADS[name]
    C = sm.switch_capacity(T, wl.num_experts, wl.capacity_factor)
    x = synth.activations(wl, T=T)
    w_r, bias = synth.router_weight(wl), synth.router_bias(wl)
    o = orc.route(x, w_r, bias, capacity=C)
    used = np.flatnonzero(np.minimum(o["counts"], C) > 0)
    w_in, w_out = synth.all_expert_weights(wl, experts=used)
    inp = dict(x=x, w_r=w_r, bias=bias, w_in=w_in, w_out=w_out)
    rep, _, _ = run_backward(orc, inp, C, 0.01, zlib.crc32(name.encode()))
    record_property("err_over_rms", rep)


def _random_inputs(rng, T, d, F, N, bias=True, w_scale=0.1):
    x = rng.standard_normal((T, d)).astype(np.float32)
    w_r = (rng.standard_normal((N, d)) * w_scale / np.sqrt(d)).astype(np.float32)
    b = (rng.standard_normal(N) * 0.2).astype(np.float32) if bias else None
    w_in = (rng.standard_normal((N, F, d)) / np.sqrt(d)).astype(np.float32)
    w_out = (rng.standard_normal((N, d, F)) / np.sqrt(F)).astype(np.float32)
    return dict(x=synth.to_bf16_bits(x), w_r=w_r, bias=b, w_in=synth.to_bf16_bits(w_in),
                w_out=synth.to_bf16_bits(w_out))


EDGE = [
    # name, T, d, F, N, C, g_aux
    ("single_expert_dense", 300, 128, 256, 1, 300, 0.5),
    ("ragged_drops", 777, 128, 192, 5, 100, 0.01),
    ("capacity_one", 400, 64, 128, 6, 1, 0.0),
    ("aux_only_weight", 500, 64, 64, 4, 200, 3.0),
    ("many_experts", 2000, 64, 128, 70, 40, 0.01),
]


@pytest.mark.parametrize("case", EDGE, ids=[c[0] for c in EDGE])
def test_backward_edge_cases(orc, case):
    name, T, d, F, N, C, g_aux = case
    inp = _random_inputs(np.random.default_rng(zlib.crc32(name.encode())), T, d, F, N)
    rep, fwd, g = run_backward(orc, inp, C, g_aux, 7)
    if N == 1:  # one expert: p = 1 identically, no router gradient at all
        assert torch.all(g["dw_r"] == 0) and torch.all(g["dbias"] == 0)


def test_backward_deterministic_and_forward_unchanged(orc):
    """Two backward calls give identical bytes, and the training forward's y equals the default forward's
    to float32 rounding (it runs the two GEMMs and the combine as separate launches)."""
    wl = synth.WORKLOADS["base8"]
    T = 1500
    C = sm.switch_capacity(T, wl.num_experts, wl.capacity_factor)
    inp = synth.inputs(wl, T=T)
    dev = {k: to_device(v) for k, v in inp.items()}
    dy = torch.randn(T, wl.d_model, device="cuda", generator=torch.Generator("cuda").manual_seed(3))
    fwd = sm.layer_fwd(dev["x"], dev["w_r"], dev["w_in"], dev["w_out"], capacity=C, flags=sm.SWITCH_FLAG_TRAINING)
    a = sm.layer_bwd(fwd, dev["x"], dev["w_r"], dev["w_in"], dev["w_out"], dy, 0.01)
    b = sm.layer_bwd(fwd, dev["x"], dev["w_r"], dev["w_in"], dev["w_out"], dy, 0.01)
    assert sm.switch_check(fwd["workspace"]) == 0
    for k in ("dx", "dw_r", "dw_in", "dw_out"):
        assert torch.equal(a[k].view(torch.int32), b[k].view(torch.int32)), k
    plain = sm.layer_fwd(dev["x"], dev["w_r"], dev["w_in"], dev["w_out"], capacity=C,
                         flags=sm.SWITCH_FLAG_FFN_TWO_LAUNCHES)
    assert torch.equal(fwd["y"].view(torch.int32), plain["y"].view(torch.int32))
    for k in ("expert", "gate", "slot", "counts", "aux"):
        assert torch.equal(fwd[k], plain[k]), k


def test_backward_requires_the_training_forward():
    wl = synth.WORKLOADS["base8"]
    T = 256
    inp = synth.inputs(wl, T=T, experts=range(2))
    dev = {k: to_device(v) for k, v in inp.items()}
    fwd = sm.layer_fwd(dev["x"], dev["w_r"], dev["w_in"], dev["w_out"], capacity_factor=1.25)
    fwd["flags"] = 0
    with pytest.raises(sm.SwitchError) as ei:
        sm.layer_bwd(fwd, dev["x"], dev["w_r"], dev["w_in"], dev["w_out"], torch.zeros(T, wl.d_model, device="cuda"))
    assert ei.value.status == 6  # SWITCH_ERR_UNSUPPORTED
