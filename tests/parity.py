"""GPU-vs-oracle comparison protocol for the Switch layer.

* expert ids must equal the oracle's on every token whose top-2 logit margin
  (oracle fp64 logits, bias included) exceeds 1e-5; near-tie tokens are
  counted and their flips reported;
* slot, counts and slot_token must equal, bit for bit, the oracle's
  capacity step run on the GPU's own ids (this checks the scan whatever the
  router did on near ties), and the oracle's own assignment when nothing
  flipped;
* aux within 1e-5 relative, gates within 1e-5 absolute of the oracle's p at
  the GPU's expert;
* outputs: max-abs error over kept rows <= 2e-2 x RMS(oracle kept rows) for
  bf16 experts, <= 1e-4 x RMS for float32; dropped rows exactly 0.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as oracle_mod
from sparse_mixture_experts_fp32_b200 import synth

MARGIN = 1e-5
TOL_BF16 = 2e-2
TOL_F32 = 1e-4
AUX_RTOL = 1e-5
GATE_ATOL = 1e-5


def to_device(a: np.ndarray | None, dev="cuda"):
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def y_to_numpy(y: torch.Tensor) -> np.ndarray:
    return y.float().cpu().numpy().astype(np.float64)


class Report(dict):
    pass


def check_routing(o: dict, g: dict, orc: oracle_mod.Oracle, N: int, C: int, T: int, check_slot_token=True) -> Report:
    """o: oracle route() result (with probs); g: numpy copies of the GPU outputs."""
    rep = Report()
    near = o["margin"] <= MARGIN
    far = ~near
    mism = np.flatnonzero((g["expert"] != o["expert"]) & far)
    assert mism.size == 0, f"{mism.size} expert ids differ on tokens with margin > {MARGIN}: {mism[:10]}"
    flips = int(((g["expert"] != o["expert"]) & near).sum())
    rep["near_ties"] = int(near.sum())
    rep["flips"] = flips
    a = orc.assign(g["expert"], N, C)
    assert np.array_equal(g["counts"], a["counts"]), "counts differ from the oracle's count of the GPU ids"
    bad = np.flatnonzero(g["slot"] != a["slot"])
    assert bad.size == 0, f"{bad.size} slots differ from the oracle's assignment of the GPU ids: {bad[:10]}"
    if check_slot_token:
        assert np.array_equal(g["slot_token"].reshape(N, C), a["slot_token"]), "slot_token differs"
    if flips == 0:
        assert np.array_equal(g["slot"], o["slot"]) and np.array_equal(g["counts"], o["counts"])
    # aux with the GPU's counts (identical to the oracle's when nothing flipped)
    aux_ref = orc.aux(T, a["counts"], o["prob_sum"]) if T > 0 else 0.0
    if T > 0:
        rel = abs(float(g["aux"]) - aux_ref) / abs(aux_ref)
        assert rel <= AUX_RTOL, f"aux {float(g['aux'])} vs {aux_ref} (rel {rel:.3e})"
        rep["aux_rel_err"] = rel
        p_at = o["probs"][np.arange(T), g["expert"]]
        gerr = float(np.abs(g["gate"].astype(np.float64) - p_at).max())
        assert gerr <= GATE_ATOL, f"gate error {gerr}"
        rep["gate_max_err"] = gerr
    rep["assign"] = a
    rep["drops"] = int((a["slot"] < 0).sum())
    return rep


def check_outputs(y_gpu: np.ndarray, rows: np.ndarray, o: dict, rep: Report, orc, x, w_in, w_out, g_expert,
                  fp32: bool) -> None:
    """Compare GPU output rows (y_gpu[r] is token rows[r]) with the oracle's, using the GPU's ids."""
    slot = rep["assign"]["slot"]
    T = slot.shape[0]
    gate = o["probs"][np.arange(T), g_expert]
    ref = orc.output_rows(rows, x, w_in, w_out, g_expert, slot, gate)
    got = y_gpu
    kept = slot[rows] >= 0
    if (~kept).any():
        assert np.all(got[~kept] == 0.0), "a dropped token has a nonzero output row"
    if kept.any():
        rms = float(np.sqrt(np.mean(ref[kept] ** 2)))
        err = float(np.abs(got[kept] - ref[kept]).max())
        tol = (TOL_F32 if fp32 else TOL_BF16) * rms
        rep["y_rms"] = rms
        rep["y_max_abs_err"] = err
        rep["y_err_over_rms"] = err / rms if rms > 0 else 0.0
        assert err <= tol, f"max-abs output error {err:.4e} > {tol:.4e} (RMS {rms:.4e})"


def oracle_route(orc, inp, C):
    return orc.route(inp["x"], inp["w_r"], inp["bias"], capacity=C, want_probs=True)


def workload_inputs(wl: synth.Workload, T=None, oracle_route_first=None, orc=None, C=None):
    """Inputs for a workload; expert weights only for experts that the oracle
    routes kept tokens to (other experts are zeros and are never read)."""
    x = synth.activations(wl, T=T)
    w_r = synth.router_weight(wl)
    bias = synth.router_bias(wl)
    inp = dict(x=x, w_r=w_r, bias=bias)
    o = orc.route(x, w_r, bias, capacity=C, want_probs=True)
    used = np.flatnonzero(np.minimum(o["counts"], C) > 0)
    inp["w_in"], inp["w_out"] = synth.all_expert_weights(wl, experts=used)
    return inp, o


# ---------------------------------------------------------------------------
# top-2 routing
# ---------------------------------------------------------------------------
def check_routing_top2(o: dict, g: dict, orc: oracle_mod.Oracle, N: int, C: int, T: int,
                       check_slot_token=True) -> Report:
    """o: oracle route_top2() result (with probs); g: numpy copies of the GPU outputs ([T, 2] per token).

    A token whose first-choice margin is <= MARGIN may swap its two choices, and
    one whose second-choice margin is <= MARGIN may pick another second choice;
    every other token's two ids must equal the oracle's.  The capacity step is
    then checked bit for bit on the GPU's own ids."""
    rep = Report()
    near1 = o["margin"][:, 0] <= MARGIN
    near2 = o["margin"][:, 1] <= MARGIN
    far = ~(near1 | near2)
    diff = (g["expert"] != o["expert"]).any(axis=1)
    mism = np.flatnonzero(diff & far)
    assert mism.size == 0, f"{mism.size} top-2 ids differ on tokens with margins > {MARGIN}: {mism[:10]}"
    rep["near_ties"] = int((~far).sum())
    rep["flips"] = int((diff & ~far).sum())
    a = orc.assign_top2(g["expert"], N, C)
    assert np.array_equal(g["counts"], a["counts"]), "counts differ from the oracle's count of the GPU ids"
    bad = np.flatnonzero((g["slot"] != a["slot"]).any(axis=1))
    assert bad.size == 0, f"{bad.size} tokens' slots differ from the oracle's assignment of the GPU ids: {bad[:10]}"
    if check_slot_token:
        assert np.array_equal(g["slot_token"].reshape(N, C), a["slot_token"]), "slot_token differs"
    if rep["flips"] == 0:
        assert np.array_equal(g["slot"], o["slot"]) and np.array_equal(g["counts"], o["counts"])
    if T > 0:
        aux_ref = orc.aux(T, a["counts_first"], o["prob_sum"])
        rel = abs(float(g["aux"]) - aux_ref) / abs(aux_ref)
        assert rel <= AUX_RTOL, f"aux {float(g['aux'])} vs {aux_ref} (rel {rel:.3e})"
        rep["aux_rel_err"] = rel
        p_at = np.take_along_axis(o["probs"], g["expert"].astype(np.int64), axis=1)
        gerr = float(np.abs(g["gate"].astype(np.float64) - p_at).max())
        assert gerr <= GATE_ATOL, f"gate error {gerr}"
        rep["gate_max_err"] = gerr
    rep["assign"] = a
    rep["dropped_choices"] = int((a["slot"] < 0).sum())
    return rep


def check_outputs_top2(y_gpu: np.ndarray, rows: np.ndarray, o: dict, rep: Report, orc, x, w_in, w_out, g_expert,
                       fp32: bool) -> None:
    """GPU output rows against the oracle's top-2 outputs computed with the GPU's ids."""
    slot = rep["assign"]["slot"]
    gate = np.take_along_axis(o["probs"], g_expert.astype(np.int64), axis=1)
    ref = orc.output_rows_top2(rows, x, w_in, w_out, g_expert, slot, gate)
    kept = (slot[rows] >= 0).any(axis=1)
    if (~kept).any():
        assert np.all(y_gpu[~kept] == 0.0), "a token with both choices dropped has a nonzero output row"
    if kept.any():
        rms = float(np.sqrt(np.mean(ref[kept] ** 2)))
        err = float(np.abs(y_gpu[kept] - ref[kept]).max())
        tol = (TOL_F32 if fp32 else TOL_BF16) * rms
        rep["y_rms"] = rms
        rep["y_max_abs_err"] = err
        rep["y_err_over_rms"] = err / rms if rms > 0 else 0.0
        assert err <= tol, f"max-abs output error {err:.4e} > {tol:.4e} (RMS {rms:.4e})"


# ---------------------------------------------------------------------------
# backward pass: per-element error bounds derived from the arithmetic
# ---------------------------------------------------------------------------
U_BF16 = 2.0 ** -8   # unit roundoff of bfloat16 (8 significant bits, round to nearest)
U_F32 = 2.0 ** -24   # unit roundoff of float32
EPS_P = 2.0 ** -18   # relative error of the float32 router probabilities and their sums


def _f64(a):
    return synth.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def backward_error_bounds(inp: dict, C: int, dy: np.ndarray, g_aux: float, route: dict) -> dict:
    """First-order bounds on |GPU - exact| for every gradient, from the rounding points of the
    CUDA path: the hidden activations H, gate * dy and the pre-activation gradient dZ enter the
    expert matmuls as bfloat16 (one rounding each, relative error <= u = 2^-8), every matmul
    accumulates in float32 (K terms: <= K * 2^-24 relative to the sum of absolute products), and
    the router's probabilities are float32 (relative error <= 2^-18).  For a dot product of a
    rounded operand with an exact one the error is at most (u + K 2^-24) times the sum of
    absolute products; the bounds below chain that through the backward's steps (magnitudes
    computed in float64 from the inputs and the oracle's routing).
    The router products run on the tensor cores over exact three-term bfloat16 splits of their
    float32 operands (products exact; float32 accumulation taken as <= 2^-23 per addition, which
    also covers truncating adders): dx's router part sums 6N split products (the three dropped
    term pairs add <= 2^-23 of |dh| |W_r|), so (12N + 3) 2^-24; dW_r sums <= Tc <= T products per
    chunk and term, then three terms and <= 64 chunks in float32, so (2T + 67) 2^-24; d bias is a
    float32 sum in token order per chunk, then over the chunks, so (T + 64) 2^-24.  These also
    bound the float32 FMA router kernels (N 2^-24 and T 2^-24).  route: oracle route() with probs."""
    x = _f64(inp["x"])
    w_in, w_out = _f64(inp["w_in"]), _f64(inp["w_out"])
    w_r = inp["w_r"].astype(np.float64)
    T, d = x.shape
    N, F, _ = w_in.shape
    p, e_of, slot = route["probs"], route["expert"], route["slot"]
    gate = p[np.arange(T), e_of]
    dy = dy.astype(np.float64)
    g_f, g_d, g_c = F * U_F32, d * U_F32, max(C, 1) * U_F32
    b = dict(dx=np.zeros((T, d)), dw_in=np.zeros((N, F, d)), dw_out=np.zeros((N, d, F)))
    err_g = np.zeros(T)                      # bound on the gate gradient's error
    for e in range(N):
        toks = np.flatnonzero((e_of == e) & (slot >= 0))
        if toks.size == 0:
            continue
        xe = x[toks]
        aw_in, aw_out = np.abs(w_in[e]), np.abs(w_out[e])
        h = np.maximum(xe @ w_in[e].T, 0.0)
        ho = h @ aw_out.T                              # |W_out| |H|: magnitude of o's terms
        err_g[toks] = (U_BF16 + g_f) * (np.abs(dy[toks]) * ho).sum(1) + g_d * np.abs(dy[toks] * (h @ w_out[e].T)).sum(1)
        de = np.abs(gate[toks, None] * dy[toks])
        mask = (xe @ w_in[e].T) > 0
        mz = (de @ aw_out) * mask                      # magnitude of dZ's terms
        b["dx"][toks] += (2 * U_BF16 + 2 * g_f + 2 * g_d) * (mz @ aw_in)
        b["dw_out"][e] = (2 * U_BF16 + g_c) * (de.T @ h)
        b["dw_in"][e] = (2 * U_BF16 + 2 * g_d + g_c) * (mz.T @ np.abs(xe))
    onehot = np.zeros((T, N))
    onehot[np.arange(T), e_of] = 1.0
    g_gate = np.zeros(T)
    kept = slot >= 0
    # exact gate gradients, for the magnitude of dp
    for e in range(N):
        toks = np.flatnonzero((e_of == e) & kept)
        if toks.size:
            o = np.maximum(x[toks] @ w_in[e].T, 0.0) @ w_out[e].T
            g_gate[toks] = (dy[toks] * o).sum(1)
    dp = g_aux * N * route["counts"][None, :] / T / T + onehot * g_gate[:, None]
    dh = p * (dp - (p * dp).sum(1, keepdims=True))
    err_dh = p * (onehot + gate[:, None]) * err_g[:, None] + \
        EPS_P * (p * np.abs(dp) + p * (p * np.abs(dp)).sum(1, keepdims=True))
    g_rdx, g_rdw, g_db = (12 * N + 3) * U_F32, (2 * T + 67) * U_F32, (T + 64) * U_F32
    b["dx"] += err_dh @ np.abs(w_r) + g_rdx * (np.abs(dh) @ np.abs(w_r))
    b["dw_r"] = err_dh.T @ np.abs(x) + g_rdw * (np.abs(dh).T @ np.abs(x))
    b["dbias"] = err_dh.sum(0) + g_db * np.abs(dh).sum(0)
    return b


def check_within_bound(name: str, got: np.ndarray, ref: np.ndarray, bound: np.ndarray, report: dict,
                       slack: float = 2.0) -> None:
    """|got - ref| <= slack * bound + a float32 floor, element by element; report the worst ratio."""
    floor = 4 * U_F32 * (np.abs(ref).max() if ref.size else 0.0) + 1e-30
    err = np.abs(got - ref)
    ratio = err / (slack * bound + floor)
    worst = float(ratio.max()) if ratio.size else 0.0
    report[name] = worst
    if worst > 1.0:
        i = np.unravel_index(int(np.argmax(ratio)), ratio.shape)
        raise AssertionError(f"{name}: error {err[i]:.3e} at {i} exceeds {slack} x bound {bound[i]:.3e} "
                             f"(got {got[i]:.6e}, exact {ref[i]:.6e})")
