"""Top-2 routing on the CUDA path (through the C ABI) against the fp64 oracle.

The classic mixture-of-experts variant of the layer: the two largest softmax
probabilities select two experts per token and weight their outputs; capacity
applies per (token, choice), first choices ranked before second choices.
Small cases compare every token and every output element; full-size cases
compare routing on every token and outputs on sampled rows.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_fp32_b200 as sm
from sparse_mixture_experts_fp32_b200 import synth
from parity import check_outputs_top2, check_routing_top2, to_device, y_to_numpy

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def orc():
    return oracle.Oracle()


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return sm.lib()


def run_top2(inp, C, flags=0):
    x = to_device(inp["x"])
    out = sm.layer_fwd_top2(x, to_device(inp["w_r"]), to_device(inp["w_in"]), to_device(inp["w_out"]), capacity=C,
                            logit_bias=to_device(inp["bias"]), flags=flags)
    assert sm.switch_check(out["workspace"]) == 0
    g = {k: out[k].cpu().numpy() for k in ("expert", "gate", "slot", "counts", "aux")}
    g["aux"] = g["aux"][0]
    return g, y_to_numpy(out["y"]), out


def top2_inputs(orc, wl, T, C):
    x = synth.activations(wl, T=T)
    w_r, bias = synth.router_weight(wl), synth.router_bias(wl)
    o = orc.route_top2(x, w_r, bias, capacity=C, want_probs=True)
    used = np.flatnonzero(np.minimum(o["counts"], C) > 0)
    w_in, w_out = synth.all_expert_weights(wl, experts=used)
    return dict(x=x, w_r=w_r, bias=bias, w_in=w_in, w_out=w_out), o


def full_check_top2(orc, wl, T, flags=0):
    C = sm.switch_capacity(T, wl.num_experts, wl.capacity_factor)
    inp, o = top2_inputs(orc, wl, T, C)
    g, y, _ = run_top2(inp, C, flags)
    rep = check_routing_top2(o, g, orc, wl.num_experts, C, T, check_slot_token=False)
    check_outputs_top2(y, np.arange(T), o, rep, orc, inp["x"], inp["w_in"], inp["w_out"], g["expert"],
                       wl.dtype == synth.F32)
    return rep


SMALL = [("tiny_fp32", 64), ("base8", 1000), ("base128_skew", 4000), ("large128", 1500), ("bigexpert64", 300)]


@pytest.mark.parametrize("name,T", SMALL, ids=[n for n, _ in SMALL])
def test_top2_layer_small_all_rows(orc, name, T, record_property):
    rep = full_check_top2(orc, synth.WORKLOADS[name], T)
    for k in ("near_ties", "flips", "dropped_choices", "aux_rel_err", "y_err_over_rms"):
        record_property(k, rep.get(k))


@pytest.mark.parametrize("name,T", [("base8", 1000), ("base128_skew", 3000), ("large128", 700)])
def test_top2_simt_router(orc, name, T):
    # the CUDA-core routers' top-2 epilogues (staged for N <= 32, tiled above)
    full_check_top2(orc, synth.WORKLOADS[name], T, flags=sm.SWITCH_FLAG_SIMT_ROUTER)


def test_top2_simt_ffn_and_one_cta_gemm(orc):
    full_check_top2(orc, synth.WORKLOADS["base8"], 900, flags=sm.SWITCH_FLAG_SIMT_FFN)
    full_check_top2(orc, synth.WORKLOADS["large128"], 900, flags=sm.SWITCH_FLAG_GEMM_1CTA)


def _random_inputs(rng, T, d, F, N, dtype, bias=True):
    x = rng.standard_normal((T, d)).astype(np.float32)
    w_r = (rng.standard_normal((N, d)) * 0.1 / np.sqrt(d)).astype(np.float32)
    b = (rng.standard_normal(N) * 0.2).astype(np.float32) if bias else None
    w_in = (rng.standard_normal((N, F, d)) / np.sqrt(d)).astype(np.float32)
    w_out = (rng.standard_normal((N, d, F)) / np.sqrt(F)).astype(np.float32)
    if dtype == "bf16":
        x, w_in, w_out = synth.to_bf16_bits(x), synth.to_bf16_bits(w_in), synth.to_bf16_bits(w_out)
    return dict(x=x, w_r=w_r, bias=b, w_in=w_in, w_out=w_out)


EDGE = [
    # name, T, d, F, N, C, dtype
    ("two_experts_no_drops", 600, 64, 128, 2, 600, "bf16"),
    ("two_experts_drops", 600, 64, 128, 2, 250, "bf16"),
    ("one_token", 1, 64, 64, 4, 1, "bf16"),
    ("ragged_tail", 1000, 128, 192, 6, 200, "bf16"),
    ("capacity_one", 500, 64, 128, 5, 1, "bf16"),
    ("max_experts", 3000, 64, 128, 256, 24, "bf16"),
    ("experts_33", 2000, 128, 128, 33, 140, "bf16"),
    ("f32_odd_shapes", 77, 33, 17, 3, 60, "f32"),
    ("f32_many_experts", 900, 48, 40, 70, 30, "f32"),
]


@pytest.mark.parametrize("case", EDGE, ids=[c[0] for c in EDGE])
def test_top2_edge_cases(orc, case):
    name, T, d, F, N, C, dt = case
    inp = _random_inputs(np.random.default_rng(zlib.crc32(name.encode())), T, d, F, N, dt)
    g, y, _ = run_top2(inp, C)
    o = orc.route_top2(inp["x"], inp["w_r"], inp["bias"], capacity=C, want_probs=True)
    rep = check_routing_top2(o, g, orc, N, C, T, check_slot_token=False)
    check_outputs_top2(y, np.arange(T), o, rep, orc, inp["x"], inp["w_in"], inp["w_out"], g["expert"], dt == "f32")


def test_top2_first_choices_are_top1_routing(orc):
    """First choices (ids, gates, slots) equal the top-1 layer's routing on the same inputs."""
    wl = synth.WORKLOADS["large128"]
    T = 3000
    inp = synth.inputs(wl, T=T, experts=range(4))
    dev = {k: to_device(v) for k, v in inp.items()}
    C = sm.switch_capacity(T, wl.num_experts, wl.capacity_factor)
    a = sm.route(dev["x"], dev["w_r"], capacity=C, d_ff=wl.d_ff)
    b = sm.route_top2(dev["x"], dev["w_r"], capacity=C, d_ff=wl.d_ff)
    assert sm.switch_check(a["workspace"]) == 0 and sm.switch_check(b["workspace"]) == 0
    assert torch.equal(b["expert"][:, 0], a["expert"])
    assert torch.equal(b["gate"][:, 0], a["gate"])
    assert torch.equal(b["slot"][:, 0], a["slot"])
    assert float(b["aux"][0]) == float(a["aux"][0])


def test_top2_entry_points_compose_to_layer():
    """route_top2 -> dispatch -> expert_ffn -> combine_top2 gives the same bytes as layer_fwd_top2 with
    the two expert GEMMs launched one after the other, and agrees with the default layer_fwd_top2
    (one persistent launch, which may split its second GEMM over d_ff) to float32 rounding."""
    wl = synth.WORKLOADS["base8"]
    T = 2000
    C = sm.switch_capacity(T, wl.num_experts, 2.0)
    inp = synth.inputs(wl, T=T)
    dev = {k: to_device(v) for k, v in inp.items()}
    ref = sm.layer_fwd_top2(dev["x"], dev["w_r"], dev["w_in"], dev["w_out"], capacity=C,
                            flags=sm.SWITCH_FLAG_FFN_TWO_LAUNCHES)
    fused = sm.layer_fwd_top2(dev["x"], dev["w_r"], dev["w_in"], dev["w_out"], capacity=C)
    assert sm.switch_check(ref["workspace"]) == 0 and sm.switch_check(fused["workspace"]) == 0
    rms = float(ref["y"].double().pow(2).mean().sqrt())
    assert float((fused["y"].double() - ref["y"].double()).abs().max()) <= 1e-4 * rms
    d = sm.layer_dims(dev["x"], dev["w_in"], capacity=C)
    ws = sm.workspace(d, "cuda")
    N, dm = wl.num_experts, wl.d_model
    r = sm.route_top2(dev["x"], dev["w_r"], capacity=C, d_ff=wl.d_ff, ws=ws)
    xbuf = torch.empty(N * C * dm, dtype=torch.bfloat16, device="cuda")
    ybuf = torch.empty(N * C * dm, dtype=torch.float32, device="cuda")
    y = torch.empty(T, dm, dtype=torch.float32, device="cuda")
    sm.switch_dispatch(d, dev["x"], r["slot_token"], r["counts"], xbuf)
    sm.switch_expert_ffn(d, xbuf, dev["w_in"], dev["w_out"], r["counts"], ybuf, ws)
    sm.switch_combine_top2(d, ybuf, r["expert"], r["slot"], r["gate"], y)
    assert sm.switch_check(ws) == 0
    for k in ("expert", "gate", "slot", "counts", "aux"):
        assert torch.equal(r[k], ref[k]), k
    assert torch.equal(y.view(torch.int32), ref["y"].view(torch.int32))


@pytest.mark.parametrize("name,T", [("base128_skew", 6000), ("base8", 3000)])
def test_top2_deterministic_bytes(name, T):
    wl = synth.WORKLOADS[name]
    inp = synth.inputs(wl, T=T, experts=range(8))
    dev = {k: to_device(v) for k, v in inp.items()}
    C = sm.switch_capacity(T, wl.num_experts, wl.capacity_factor)
    a = sm.layer_fwd_top2(dev["x"], dev["w_r"], dev["w_in"], dev["w_out"], capacity=C, logit_bias=dev["bias"])
    b = sm.layer_fwd_top2(dev["x"], dev["w_r"], dev["w_in"], dev["w_out"], capacity=C, logit_bias=dev["bias"])
    for k in ("expert", "gate", "slot", "counts", "aux"):
        assert torch.equal(a[k], b[k]), k
    assert torch.equal(a["y"].view(torch.int32), b["y"].view(torch.int32))


def _sample_rows(slot, n_kept=256, n_any=64, seed=0):
    rng = np.random.default_rng(seed)
    kept = np.flatnonzero((slot >= 0).any(axis=1))
    pick = rng.choice(kept, size=min(n_kept, kept.size), replace=False) if kept.size else np.array([], np.int64)
    extra = rng.choice(slot.shape[0], size=min(n_any, slot.shape[0]), replace=False)
    return np.unique(np.concatenate([pick, extra]).astype(np.int64))


@pytest.mark.parametrize("name", ["base8", "large128"])
def test_top2_full_size(orc, name, record_property):
    """The workload at full size: routing on every token, outputs on sampled rows,
    every both-dropped row exactly zero (checked on the device)."""
    wl = synth.WORKLOADS[name]
    T, N = wl.T, wl.num_experts
    C = sm.switch_capacity(T, N, wl.capacity_factor)
    inp, o = top2_inputs(orc, wl, T, C)
    g, _, out = None, None, None
    x = to_device(inp["x"])
    out = sm.layer_fwd_top2(x, to_device(inp["w_r"]), to_device(inp["w_in"]), to_device(inp["w_out"]), capacity=C,
                            logit_bias=to_device(inp["bias"]))
    assert sm.switch_check(out["workspace"]) == 0
    g = {k: out[k].cpu().numpy() for k in ("expert", "gate", "slot", "counts", "aux")}
    g["aux"] = g["aux"][0]
    rep = check_routing_top2(o, g, orc, N, C, T, check_slot_token=False)
    both = torch.from_numpy((rep["assign"]["slot"] < 0).all(axis=1)).cuda()
    assert torch.all(out["y"][both] == 0)
    rows = _sample_rows(rep["assign"]["slot"])
    y_rows = out["y"][torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
    check_outputs_top2(y_rows, rows, o, rep, orc, inp["x"], inp["w_in"], inp["w_out"], g["expert"], False)
    record_property("report", {k: rep.get(k) for k in ("near_ties", "flips", "dropped_choices", "aux_rel_err",
                                                       "y_err_over_rms")})
