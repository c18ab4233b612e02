"""Backward pass of the layer on the CUDA path (through the C ABI) against the
fp64 backward oracle, element by element.

The loss is L = sum(y * dy) + g_aux * aux with a seeded upstream gradient dy.
The expert GEMMs take bfloat16 operands (the hidden activations H, gate * dy
and the pre-activation gradient dZ, each rounded once) and accumulate in
float32; the router products run on the tensor cores over exact three-term
bfloat16 splits of their float32 operands (or, with SWITCH_FLAG_SIMT_ROUTER,
as float32 FMA kernels).  The tolerance is derived from that
arithmetic, element by element: every gradient must lie within twice the
first-order floating-point error bound of its computation (for each dot
product, the unit roundoffs of its rounded operands plus K float32 roundings,
times the sum of the absolute values of its terms; parity.backward_error_bounds).
A test with exactly representable data checks the expert path to float32
exactness.  Routing is the GPU forward's own and must equal the oracle's.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_fp32_b200 as sm
from sparse_mixture_experts_fp32_b200 import synth
from parity import backward_error_bounds, check_within_bound, to_device

pytestmark = pytest.mark.gpu

@pytest.fixture(scope="module")
def orc():
    return oracle.Oracle()


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return sm.lib()


def run_backward(orc, inp, C, g_aux, seed, check_bias=True, flags=0):
    T, d = inp["x"].shape
    rng = np.random.default_rng(seed)
    dy = rng.standard_normal((T, d)).astype(np.float32)
    dev = {k: to_device(v) for k, v in inp.items()}
    fwd = sm.layer_fwd(dev["x"], dev["w_r"], dev["w_in"], dev["w_out"], capacity=C, logit_bias=dev["bias"],
                       flags=sm.SWITCH_FLAG_TRAINING | flags)
    g = sm.layer_bwd(fwd, dev["x"], dev["w_r"], dev["w_in"], dev["w_out"], torch.from_numpy(dy).cuda(), g_aux,
                     logit_bias=dev["bias"])
    assert sm.switch_check(fwd["workspace"]) == 0
    o = orc.route(inp["x"], inp["w_r"], inp["bias"], capacity=C, want_probs=True)
    assert np.array_equal(fwd["expert"].cpu().numpy(), o["expert"]), "routing differs (near tie in a gradient case)"
    ref = orc.layer_bwd(inp["x"], inp["w_r"], inp["w_in"], inp["w_out"], dy.astype(np.float64), g_aux,
                        bias=inp["bias"], capacity=C)
    bound = backward_error_bounds(inp, C, dy, g_aux, o)
    rep = {}
    names = ["dx", "dw_r", "dw_in", "dw_out"] + (["dbias"] if check_bias and inp["bias"] is not None else [])
    for k in names:
        check_within_bound(k, g[k].double().cpu().numpy(), ref[k], bound[k], rep)
    # experts without kept tokens get exactly zero weight gradients
    kept = np.minimum(o["counts"], C) > 0
    if (~kept).any():
        idle = torch.from_numpy(~kept).cuda()
        assert torch.all(g["dw_in"][idle] == 0) and torch.all(g["dw_out"][idle] == 0)
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
    record_property("worst_error_over_bound", rep)


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
    # tensor-core dW_r over 61 chunks of 1152 tokens (ragged last chunk), dx over 274 row tiles
    ("many_token_chunks", 70000, 64, 64, 70, 1300, 0.01),
]


@pytest.mark.parametrize("case", EDGE, ids=[c[0] for c in EDGE])
def test_backward_edge_cases(orc, case):
    name, T, d, F, N, C, g_aux = case
    inp = _random_inputs(np.random.default_rng(zlib.crc32(name.encode())), T, d, F, N)
    rep, fwd, g = run_backward(orc, inp, C, g_aux, 7)
    if N == 1:  # one expert: p = 1 identically, no router gradient at all
        assert torch.all(g["dw_r"] == 0) and torch.all(g["dbias"] == 0)


@pytest.mark.parametrize("name,T", [("base128_skew", 3000), ("base8", 600)])
def test_backward_simt_router(orc, name, T):
    """The float32 FMA router products (SWITCH_FLAG_SIMT_ROUTER) against the oracle, next to the
    tensor-core router products on the same inputs: both within their bounds.  The flag also selects
    the forward's float32 FMA router; where that gives the same gates bit for bit (N <= 32 runs the
    same router either way), the expert-path gradients are identical too."""
    wl = synth.WORKLOADS[name]
    C = sm.switch_capacity(T, wl.num_experts, wl.capacity_factor)
    x = synth.activations(wl, T=T)
    w_r, bias = synth.router_weight(wl), synth.router_bias(wl)
    used = np.flatnonzero(np.minimum(orc.route(x, w_r, bias, capacity=C)["counts"], C) > 0)
    w_in, w_out = synth.all_expert_weights(wl, experts=used)
    inp = dict(x=x, w_r=w_r, bias=bias, w_in=w_in, w_out=w_out)
    _, f_simt, g_simt = run_backward(orc, inp, C, 0.01, 5, flags=sm.SWITCH_FLAG_SIMT_ROUTER)
    _, f_tc, g_tc = run_backward(orc, inp, C, 0.01, 5)
    if torch.equal(f_simt["gate"], f_tc["gate"]):
        for k in ("dw_in", "dw_out"):
            assert torch.equal(g_simt[k], g_tc[k]), k
    else:
        assert wl.num_experts > 32


def exact_problem(rng, T=400, d=128, F=192, N=4):
    """Sparse dyadic data whose every rounding is exact.  x, dy in {-1, 0, 1}; two entries of +-1/8
    per row of W_in[e] and of W_out[e], so pre-activations, hidden values and pre-activation
    gradients are small multiples of 1/8 (exact in bfloat16) and every sum is exact in float32.
    The router is one-hot with a margin of 300: x[t, :N] is the one-hot code of token t's expert and
    W_r = 300 I on those columns, so p is exactly 1 at the chosen expert and 0 elsewhere in float32
    (exp(-300) underflows) and equal to 1 in float64: the gate is 1, the router gradient vanishes."""
    x = rng.integers(-1, 2, size=(T, d)).astype(np.float32)
    ids = rng.integers(0, N, size=T)
    x[:, :N] = 0.0
    x[np.arange(T), ids] = 1.0
    dy = rng.integers(-1, 2, size=(T, d)).astype(np.float32)
    w_r = np.zeros((N, d), np.float32)
    w_r[np.arange(N), np.arange(N)] = 300.0
    w_in = np.zeros((N, F, d), np.float32)
    w_out = np.zeros((N, d, F), np.float32)
    for e in range(N):
        for j in range(F):
            w_in[e, j, rng.choice(d, 2, replace=False)] = rng.choice([-0.125, 0.125], 2)
        for k in range(d):
            w_out[e, k, rng.choice(F, 2, replace=False)] = rng.choice([-0.125, 0.125], 2)
    inp = dict(x=synth.to_bf16_bits(x), w_r=w_r, bias=None, w_in=synth.to_bf16_bits(w_in),
               w_out=synth.to_bf16_bits(w_out))
    return inp, dy, ids


@pytest.mark.parametrize("capacity", [400, 70])
def test_backward_exact_arithmetic(orc, capacity):
    """With exactly representable operands and sums the GPU's expert-path gradients equal the
    oracle's exactly: the per-expert indexing, the slot-to-token scatter of dx, the ReLU masks, the
    token-major (MN-major) operand reads and the zeroing past each expert's kept tokens are pinned
    without any tolerance (with capacity 70 some tokens are dropped; theirs and the router's
    gradients are 0)."""
    inp, dy, ids = exact_problem(np.random.default_rng(21))
    T, d = dy.shape
    dev = {k: to_device(v) for k, v in inp.items()}
    fwd = sm.layer_fwd(dev["x"], dev["w_r"], dev["w_in"], dev["w_out"], capacity=capacity,
                       flags=sm.SWITCH_FLAG_TRAINING)
    g = sm.layer_bwd(fwd, dev["x"], dev["w_r"], dev["w_in"], dev["w_out"], torch.from_numpy(dy).cuda(), 0.5)
    assert sm.switch_check(fwd["workspace"]) == 0
    assert np.array_equal(fwd["expert"].cpu().numpy(), ids) and torch.all(fwd["gate"] == 1.0)
    ref = orc.layer_bwd(inp["x"], inp["w_r"], inp["w_in"], inp["w_out"], dy.astype(np.float64), 0.5,
                        capacity=capacity)
    for k in ("dw_in", "dw_out"):
        assert np.array_equal(g[k].double().cpu().numpy(), ref[k]), k
    # the oracle's router probabilities off the chosen expert are ~1e-130 instead of 0: its router
    # terms (dW_r, and all of a dropped token's dx) are that small, the GPU's exactly 0
    assert np.allclose(g["dx"].double().cpu().numpy(), ref["dx"], rtol=0, atol=1e-100)
    assert np.abs(ref["dw_r"]).max() < 1e-100 and torch.all(g["dw_r"] == 0)


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
