"""Checks that pin the fp64 oracle to facts fixed outside the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError
when the oracle disagrees with a worked example printed by the sources, a
closed form, an invariant, a special case that reduces to a library routine,
or brute force on tiny inputs.  The same functions run against the real
oracle (``test_oracle_pins.py``) and against deliberately broken copies of it
(``test_oracle_mutants.py``), which shows that each plausible mistake is
caught by at least one pin.
"""
from __future__ import annotations

import itertools
import json
from pathlib import Path

import numpy as np
import scipy.special
import scipy.stats

GOLDEN = Path(__file__).resolve().parent / "golden"


def golden(name: str) -> dict:
    return json.loads((GOLDEN / name).read_text())


def _one_hot_routing(assignment, N, scale=4.0):
    """Inputs whose router logits are scale * one_hot(assignment[t]): x[t] = e_(a_t), W_r = scale * I."""
    T = len(assignment)
    x = np.zeros((T, N), dtype=np.float32)
    x[np.arange(T), assignment] = 1.0
    w_r = (scale * np.eye(N)).astype(np.float32)
    return x, w_r


def _identity_experts(N, d):
    """Experts with W_in = W_out = I, so that E(x) = ReLU(x)."""
    eye = np.eye(d, dtype=np.float32)
    return np.stack([eye] * N), np.stack([eye] * N)


def _random_problem(rng, T, d, F, N, with_bias=True):
    x = rng.standard_normal((T, d)).astype(np.float32)
    w_r = (rng.standard_normal((N, d)) * 0.5).astype(np.float32)
    bias = (rng.standard_normal(N) * 0.3).astype(np.float32) if with_bias else None
    w_in = (rng.standard_normal((N, F, d)) / np.sqrt(d)).astype(np.float32)
    w_out = (rng.standard_normal((N, d, F)) / np.sqrt(F)).astype(np.float32)
    return x, w_r, bias, w_in, w_out


# --------------------------------------------------------------------------
# Worked examples printed by the sources
# --------------------------------------------------------------------------

def pin_capacity_examples(o):
    for case in golden("capacity_examples.json")["cases"]:
        got = o.capacity(case["T"], case["N"], case["c"])
        assert got == case["C"], (case, got)


def pin_workload_capacities(o):
    # C = ceil(T / N * c) at the five workload shapes (all exact integers).
    for T, N, c, C in [(64, 4, 1.0, 16), (8192, 8, 1.25, 1280), (65536, 128, 1.0, 512),
                       (131072, 128, 1.25, 1280), (32768, 64, 0.5, 256), (32768, 64, 1.0, 512),
                       (32768, 64, 1.25, 640), (32768, 64, 2.0, 1024)]:
        assert o.capacity(T, N, c) == C, (T, N, c)
    # Non-integer quotients round up: 10 / 3 -> 4, 7 / 2 * 1.1 = 3.85 -> 4.
    assert o.capacity(10, 3, 1.0) == 4
    assert o.capacity(7, 2, 1.1) == 4
    assert o.capacity(1, 64, 0.5) == 1


def pin_overflow_16tok(o):
    g = golden("overflow_16tok.json")
    expert = np.array(g["expert"], dtype=np.int32)
    a = o.assign(expert, g["N"], o.capacity(len(expert), g["N"], g["c"]))
    assert a["counts"].tolist() == g["counts"]
    dropped = np.flatnonzero(a["slot"] < 0).tolist()
    assert dropped == g["dropped_tokens"], dropped
    assert int((a["slot"] >= 0).sum()) == g["kept"]


def pin_overflow_16tok_routed(o):
    # The same example driven through the router: one-hot inputs make the
    # logits select the listed experts.
    g = golden("overflow_16tok.json")
    x, w_r = _one_hot_routing(g["expert"], g["N"])
    r = o.route(x, w_r, capacity_factor=g["c"])
    assert r["capacity"] == g["capacity"]
    assert r["expert"].tolist() == g["expert"]
    assert np.flatnonzero(r["slot"] < 0).tolist() == g["dropped_tokens"]


def pin_p1_moe_layer_example(o):
    g = golden("p1_moe_layer_example.json")
    a = o.assign(np.array(g["expert"], dtype=np.int32), g["N"], g["capacity"])
    for e, kept in enumerate(g["kept_by_expert"]):
        assert a["slot_token"][e].tolist() == kept, (e, a["slot_token"][e])


def pin_byhand_overflow(o):
    g = golden("byhand_5tok.json")
    rows = g["switch_matrix_rows"]
    w_r = np.array([rows["A"], rows["B"], rows["C"]], dtype=np.float32)
    z = np.array(g["Z"], dtype=np.float32)
    h = o.router_logits(z, w_r)
    assert h[4].tolist() == g["gate_values_Z5"]
    w_in, w_out = _identity_experts(3, 3)
    r = o.layer_fwd(z, w_r, w_in, w_out, capacity=g["capacity"])
    assert r["expert"].tolist() == g["expert"]
    assert r["slot"].tolist() == g["slot"]
    assert r["counts"].tolist() == g["counts"]
    # The dropped feature gets a zero layer output, so x + y passes it through unchanged.
    for t in g["dropped"]:
        assert np.all(r["y"][t] == 0.0)
        assert np.array_equal(z[t] + r["y"][t], z[t])
    kept = [t for t in range(5) if t not in g["dropped"]]
    assert all(np.any(r["y"][t] != 0.0) for t in kept)


def pin_p1_softmax_table(o):
    g = golden("p1_softmax_table.json")
    p = np.array(g["probs"], dtype=np.float64)
    # Logits whose softmax is the printed row: h = ln p (a zero probability
    # becomes a logit so low that its exponential underflows to 0).
    h = np.where(p > 0, np.log(np.where(p > 0, p, 1.0)), -1000.0)
    r = o.softmax_top1(h, want_probs=True)
    assert r["expert"].tolist() == g["selected"]
    assert np.allclose(r["probs"], p, rtol=0, atol=1e-15)
    counts = np.bincount(r["expert"], minlength=4).astype(np.int32)
    assert np.allclose(counts / 5.0, g["derived_f"], atol=0)
    assert np.allclose(r["prob_sum"] / 5.0, g["derived_P"], atol=1e-15)
    assert abs(o.aux(5, counts, r["prob_sum"]) - g["derived_aux"]) < 1e-12


def pin_p1_aux_tables(o):
    for case in golden("p1_aux_tables.json")["cases"]:
        got = o.aux(case["T"], np.array(case["counts"], np.int32), np.array(case["prob_sum"], np.float64))
        assert abs(got - case["aux"]) < 1e-12, (case["name"], got)
        assert abs(got / 4 - case["sum_fP"]) < 1e-12


def pin_kasblo_gate(o):
    g = golden("kasblo_gate_063.json")
    p = np.array(g["probs"], dtype=np.float64)
    # One token, d = N = 4; x = e_0 and W_r[:, 0] = ln p gives logits ln p.
    x = np.zeros((1, 4), dtype=np.float32)
    x[0, 0] = 1.0
    w_r = np.zeros((4, 4), dtype=np.float32)
    w_r[:, 0] = np.log(p).astype(np.float32)
    w_in, w_out = _identity_experts(4, 4)
    r = o.layer_fwd(x, w_r, w_in, w_out, capacity=1)
    assert r["expert"][0] == g["selected"]
    assert abs(r["gate"][0] - g["gate"]) < 1e-6
    # E(x) = ReLU(e_0) = e_0, so y = 0.63 * e_0.
    assert np.allclose(r["y"][0], [r["gate"][0], 0, 0, 0], atol=0)
    assert abs(r["y"][0][0] - 0.63) < 1e-6


# --------------------------------------------------------------------------
# Closed forms, special cases and invariants
# --------------------------------------------------------------------------

def pin_zero_router_uniform(o):
    # W_r = 0: every p_i = 1/N so P is uniform and aux = 1; all logits tie and
    # the lowest index wins, so every token goes to expert 0, C are kept.
    T, d, N = 40, 8, 5
    x = np.random.default_rng(1).standard_normal((T, d)).astype(np.float32)
    r = o.route(x, np.zeros((N, d), np.float32), capacity_factor=1.0)
    C = r["capacity"]
    assert C == 8
    assert r["expert"].tolist() == [0] * T
    assert r["counts"].tolist() == [T] + [0] * (N - 1)
    assert int((r["slot"] >= 0).sum()) == C and int((r["slot"] < 0).sum()) == T - C
    assert r["slot"][:C].tolist() == list(range(C))
    assert np.allclose(r["gate"], 1.0 / N, rtol=0, atol=1e-15)
    assert abs(r["aux"] - 1.0) < 1e-12


def pin_balanced_routing_aux_one(o):
    # Each expert receives exactly T/N tokens: f is uniform, so aux = 1 for any P.
    N, m = 4, 6
    assignment = np.tile(np.arange(N), m)
    np.random.default_rng(2).shuffle(assignment)
    x, w_r = _one_hot_routing(assignment, N, scale=3.0)
    w_r[0, 0] += 1.0  # make P non-uniform
    r = o.route(x, w_r, capacity_factor=1.0)
    assert r["counts"].tolist() == [m] * N
    assert not np.allclose(r["prob_sum"], r["prob_sum"][0])
    assert abs(r["aux"] - 1.0) < 1e-12


def pin_single_expert_is_dense_ffn(o):
    # N = 1: p = 1, gate = 1, C = ceil(T * c) = T at c = 1, nothing dropped,
    # so the layer is the dense FFN ReLU(x W_in^T) W_out^T (numpy reference).
    rng = np.random.default_rng(3)
    x, w_r, bias, w_in, w_out = _random_problem(rng, 20, 12, 24, 1)
    r = o.layer_fwd(x, w_r, w_in, w_out, bias=bias, capacity_factor=1.0)
    dense = np.maximum(x.astype(np.float64) @ w_in[0].astype(np.float64).T, 0.0) @ w_out[0].astype(np.float64).T
    assert r["capacity"] == 20
    assert np.all(r["gate"] == 1.0) and np.all(r["slot"] == np.arange(20))
    assert np.allclose(r["y"], dense, rtol=1e-12, atol=1e-12)
    assert abs(r["aux"] - 1.0) < 1e-12


def pin_logits_match_numpy(o):
    # h = x W_r^T + b, against numpy's float64 matrix product.
    rng = np.random.default_rng(4)
    x, w_r, bias, _, _ = _random_problem(rng, 33, 17, 4, 5)
    h = o.router_logits(x, w_r, bias)
    ref = x.astype(np.float64) @ w_r.astype(np.float64).T + bias.astype(np.float64)
    assert np.allclose(h, ref, rtol=1e-13, atol=1e-13)


def pin_bf16_loads_exact(o):
    # bfloat16 inputs convert exactly: the same values given as float32 and as
    # bf16 bit patterns give bit-identical logits.
    rng = np.random.default_rng(5)
    vals = rng.standard_normal((9, 16)).astype(np.float32)
    bits = vals.view(np.uint32) >> np.uint32(16)
    as_f32 = (bits << np.uint32(16)).view(np.float32)
    as_bf16 = bits.astype(np.uint16)
    w_r = rng.standard_normal((3, 16)).astype(np.float32)
    assert np.array_equal(o.router_logits(as_f32, w_r), o.router_logits(as_bf16, w_r))


def pin_softmax_matches_scipy(o):
    rng = np.random.default_rng(6)
    h = rng.standard_normal((50, 7)) * 3.0
    r = o.softmax_top1(h, want_probs=True)
    ref = scipy.special.softmax(h, axis=1)
    assert np.allclose(r["probs"], ref, rtol=1e-13, atol=1e-15)
    assert np.array_equal(r["expert"], np.argmax(h, axis=1))
    assert np.allclose(r["gate"], ref[np.arange(50), r["expert"]], rtol=1e-13)
    assert np.allclose(r["prob_sum"], ref.sum(axis=0), rtol=1e-13)
    srt = np.sort(h, axis=1)
    assert np.allclose(r["margin"], srt[:, -1] - srt[:, -2], rtol=0, atol=1e-15)


def pin_ties_lowest_index(o):
    h = np.array([[1.0, 3.0, 3.0, 0.0], [2.0, 2.0, 2.0, 2.0], [0.0, 0.0, 5.0, 5.0]])
    r = o.softmax_top1(h)
    assert r["expert"].tolist() == [1, 0, 2]
    assert r["margin"].tolist() == [0.0, 0.0, 0.0]


def pin_dense_masked_formulation(o):
    # A second formulation, in numpy: run every expert on every token, then
    # keep, per expert, the first C tokens (in token order) whose argmax is
    # that expert, and scale by the selected probability.
    for seed, (T, d, F, N, C) in enumerate([(40, 8, 16, 3, 10), (64, 6, 10, 5, 9), (17, 4, 8, 2, 17)]):
        rng = np.random.default_rng(100 + seed)
        x, w_r, bias, w_in, w_out = _random_problem(rng, T, d, F, N)
        r = o.layer_fwd(x, w_r, w_in, w_out, bias=bias, capacity=C)
        x64 = x.astype(np.float64)
        h = x64 @ w_r.astype(np.float64).T + bias.astype(np.float64)
        p = scipy.special.softmax(h, axis=1)
        ids = np.argmax(p, axis=1)
        every = np.stack([np.maximum(x64 @ w_in[i].astype(np.float64).T, 0) @ w_out[i].astype(np.float64).T
                          for i in range(N)])
        y = np.zeros((T, d))
        for i in range(N):
            chosen = np.flatnonzero(ids == i)[:C]
            y[chosen] = p[chosen, i][:, None] * every[i, chosen]
        assert np.array_equal(r["expert"], ids)
        assert np.allclose(r["y"], y, rtol=1e-12, atol=1e-13), np.abs(r["y"] - y).max()
        f = np.bincount(ids, minlength=N) / T
        assert abs(r["aux"] - N * np.dot(f, p.mean(axis=0))) < 1e-12


def pin_brute_force_assignment(o):
    # Every assignment of T tokens to N experts, every capacity: the kept
    # tokens of each expert are exactly its first C tokens in token order.
    for T, N in [(6, 3), (8, 2), (4, 4)]:
        for assignment in itertools.product(range(N), repeat=T):
            expert = np.array(assignment, dtype=np.int32)
            for C in range(1, T + 1):
                a = o.assign(expert, N, C)
                for e in range(N):
                    mine = [t for t in range(T) if assignment[t] == e]
                    assert a["counts"][e] == len(mine)
                    kept = mine[:C]
                    assert a["slot_token"][e].tolist() == kept + [-1] * (C - len(kept))
                    for s, t in enumerate(mine):
                        assert a["slot"][t] == (s if s < C else -1)


def pin_invariants_random(o):
    rng = np.random.default_rng(7)
    T, d, F, N = 300, 16, 32, 6
    x, w_r, bias, w_in, w_out = _random_problem(rng, T, d, F, N)
    r = o.layer_fwd(x, w_r, w_in, w_out, bias=bias, capacity_factor=0.8, want_probs=True)
    C = r["capacity"]
    assert C == 40
    assert int(r["counts"].sum()) == T
    assert np.allclose(r["probs"].sum(axis=1), 1.0, atol=1e-14)
    assert np.all(r["gate"] >= 1.0 / N - 1e-15) and np.all(r["gate"] <= 1.0)
    kept = np.minimum(r["counts"], C)
    for e in range(N):
        toks = np.flatnonzero((r["expert"] == e) & (r["slot"] >= 0))
        assert len(toks) == kept[e]
        assert r["slot"][toks].tolist() == list(range(kept[e]))
    assert int((r["slot"] < 0).sum()) == int(np.maximum(r["counts"] - C, 0).sum())
    assert np.all(r["y"][r["slot"] < 0] == 0.0)


def pin_permutation_equivariance(o):
    # With no drops, permuting the tokens permutes ids, gates and outputs and
    # leaves counts and aux unchanged.
    rng = np.random.default_rng(8)
    T, d, F, N = 48, 8, 12, 4
    x, w_r, bias, w_in, w_out = _random_problem(rng, T, d, F, N)
    perm = rng.permutation(T)
    a = o.layer_fwd(x, w_r, w_in, w_out, bias=bias, capacity=T)
    b = o.layer_fwd(x[perm], w_r, w_in, w_out, bias=bias, capacity=T)
    assert np.array_equal(a["expert"][perm], b["expert"])
    assert np.array_equal(a["counts"], b["counts"])
    assert np.allclose(a["gate"][perm], b["gate"], rtol=1e-15, atol=0)
    assert np.allclose(a["y"][perm], b["y"], rtol=1e-13, atol=1e-15)
    assert abs(a["aux"] - b["aux"]) < 1e-12


def pin_relu_and_gate_closed_form(o):
    # Identity experts: y = gate * ReLU(x) exactly, for kept tokens.
    rng = np.random.default_rng(9)
    T, N = 12, 3
    x = rng.standard_normal((T, N)).astype(np.float32)
    w_r = (rng.standard_normal((N, N))).astype(np.float32)
    w_in, w_out = _identity_experts(N, N)
    r = o.layer_fwd(x, w_r, w_in, w_out, capacity=T)
    ref = r["gate"][:, None] * np.maximum(x.astype(np.float64), 0.0)
    assert np.array_equal(r["y"], ref)


def pin_expert_weight_layout(o):
    # W_in[e] is [F, d] (row j feeds hidden unit j) and W_out[e] is [d, F]
    # (row k produces output k): a single nonzero entry in each shows where
    # the product goes.
    d, F = 3, 5
    x = np.array([[0.0, 2.0, 0.0]], dtype=np.float32)
    w_in = np.zeros((1, F, d), np.float32)
    w_out = np.zeros((1, d, F), np.float32)
    w_in[0, 4, 1] = 3.0   # hidden unit 4 = 3 * x[1] = 6
    w_out[0, 0, 4] = 0.5  # output 0 = 0.5 * hidden 4 = 3
    r = o.layer_fwd(x, np.zeros((1, d), np.float32), w_in, w_out, capacity=1)
    assert r["y"][0].tolist() == [3.0, 0.0, 0.0]


# --------------------------------------------------------------------------
# Top-2 routing (the classic mixture-of-experts variant)
# --------------------------------------------------------------------------

def _logits_of_probs(p):
    """Logits whose softmax is the given row (a zero probability becomes a logit whose exponential is 0)."""
    p = np.asarray(p, dtype=np.float64)
    return np.where(p > 0, np.log(np.where(p > 0, p, 1.0)), -1000.0)


def _top2_priority_definition(first, second, N, C):
    """Set definition of the top-2 capacity step: the assignments (t, first_t) for
    every t in token order, then (t, second_t) for every t; each expert keeps its
    first C assignments of that list."""
    T = len(first)
    order = [(t, 0, first[t]) for t in range(T)] + [(t, 1, second[t]) for t in range(T)]
    slot = np.full((T, 2), -1, dtype=np.int64)
    holders = {e: [] for e in range(N)}
    for t, c, e in order:
        if len(holders[e]) < C:
            slot[t, c] = len(holders[e])
        holders[e].append(t)
    counts = [len(holders[e]) for e in range(N)]
    kept = {e: holders[e][:C] for e in range(N)}
    return slot, counts, kept


def pin_top2_p1_softmax_table(o):
    g = golden("p1_top2_table.json")
    h = _logits_of_probs(g["probs"])
    r = o.softmax_top2(h, want_probs=True)
    assert r["expert"][:, 0].tolist() == g["ours_first"]
    assert r["expert"][:, 1].tolist() == g["ours_second"]
    assert np.allclose(r["gate"], g["ours_gates"], rtol=0, atol=1e-15)
    a = o.assign_top2(r["expert"], 4, g["capacity"])
    assert a["slot"].tolist() == g["ours_slots"]
    assert a["counts"].tolist() == g["ours_counts"]
    assert a["counts_first"].tolist() == g["ours_counts_first"]
    assert abs(o.aux(5, a["counts_first"], r["prob_sum"]) - g["derived_aux"]) < 1e-12


def pin_top2_lps_hospital(o):
    # Three experts with W_in = I and W_out = s_i I, so E_i(x) = s_i ReLU(x) tells
    # the experts apart; logits ln p on one token give y = (0.6 s_0 + 0.3 s_1) ReLU(x).
    g = golden("lps_top2_hospital.json")
    p = np.array(g["probs"])
    d = 3
    x = np.array([[1.0, 2.0, -1.0]], dtype=np.float32)
    scales = [1.0, 10.0, 100.0]
    eye = np.eye(d, dtype=np.float32)
    w_in = np.stack([eye] * 3)
    w_out = np.stack([np.float32(s) * eye for s in scales])
    # x has d = 3 features; W_r maps them to ln p: W_r[i] = ln(p_i) * e_0 / x[0]
    w_r = np.zeros((3, d), dtype=np.float32)
    w_r[:, 0] = np.log(p).astype(np.float32)
    r = o.layer_fwd_top2(x, w_r, w_in, w_out, capacity=1)
    assert r["expert"][0].tolist() == g["selected"]
    assert np.allclose(r["gate"][0], g["weights"], atol=1e-7)
    w0, w1 = r["gate"][0]
    relu = np.maximum(x[0].astype(np.float64), 0.0)
    assert np.allclose(r["y"][0], (w0 * scales[0] + w1 * scales[1]) * relu, rtol=1e-15, atol=0)
    assert abs(r["y"][0][1] - 2.0 * (0.6 * 1.0 + 0.3 * 10.0)) < 1e-5


def pin_top2_matches_argsort(o):
    # Top-2 against numpy's stable descending sort (ties keep index order), the
    # gates against scipy's softmax, the margins against the sorted logits.
    rng = np.random.default_rng(20)
    h = rng.standard_normal((80, 6)) * 2.0
    h[:5] = np.round(h[:5])  # some exact ties
    h[5] = [1.0, 1.0, 1.0, 0.0, 1.0, 0.0]
    r = o.softmax_top2(h, want_probs=True)
    order = np.argsort(-h, axis=1, kind="stable")
    assert np.array_equal(r["expert"], order[:, :2])
    ref = scipy.special.softmax(h, axis=1)
    assert np.allclose(r["gate"], np.take_along_axis(ref, order[:, :2], axis=1), rtol=1e-13, atol=1e-15)
    srt = -np.sort(-h, axis=1)
    assert np.allclose(r["margin"][:, 0], srt[:, 0] - srt[:, 1], rtol=0, atol=1e-15)
    assert np.allclose(r["margin"][:, 1], srt[:, 1] - srt[:, 2], rtol=0, atol=1e-15)
    assert np.allclose(r["prob_sum"], ref.sum(axis=0), rtol=1e-13)


def pin_top2_first_choice_is_top1(o):
    # First choices, their gates, margins and slots are those of top-1 routing
    # (first choices rank before every second choice), and aux is unchanged.
    rng = np.random.default_rng(21)
    x, w_r, bias, _, _ = _random_problem(rng, 200, 10, 4, 5)
    for C in (7, 30, 200):
        a = o.route(x, w_r, bias, capacity=C)
        b = o.route_top2(x, w_r, bias, capacity=C)
        assert np.array_equal(b["expert"][:, 0], a["expert"])
        assert np.array_equal(b["gate"][:, 0], a["gate"])
        assert np.array_equal(b["margin"][:, 0], a["margin"])
        assert np.array_equal(b["slot"][:, 0], a["slot"])
        assert np.array_equal(b["counts_first"], a["counts"])
        assert b["aux"] == a["aux"]


def pin_top2_brute_force_assignment(o):
    # Every (first, second) choice with first != second for every token, every
    # capacity, against the set definition of the priority order.
    for T, N in [(4, 3), (3, 4)]:
        pairs = [(a, b) for a in range(N) for b in range(N) if a != b]
        for combo in itertools.product(pairs, repeat=T):
            expert = np.array(combo, dtype=np.int32)
            first, second = [c[0] for c in combo], [c[1] for c in combo]
            for C in range(1, 2 * T + 1):
                a = o.assign_top2(expert, N, C)
                slot, counts, kept = _top2_priority_definition(first, second, N, C)
                assert a["slot"].tolist() == slot.tolist(), (combo, C)
                assert a["counts"].tolist() == counts
                assert a["counts_first"].tolist() == np.bincount(first, minlength=N).tolist()
                for e in range(N):
                    assert a["slot_token"][e].tolist() == kept[e] + [-1] * (C - len(kept[e]))


def pin_top2_dense_masked_formulation(o):
    # numpy: every expert on every token, the two largest probabilities (stable
    # sort), the priority-list capacity, then the probability-weighted sum.
    for seed, (T, d, F, N, C) in enumerate([(40, 8, 16, 4, 12), (30, 6, 10, 3, 9), (25, 4, 8, 5, 50)]):
        rng = np.random.default_rng(120 + seed)
        x, w_r, bias, w_in, w_out = _random_problem(rng, T, d, F, N)
        r = o.layer_fwd_top2(x, w_r, w_in, w_out, bias=bias, capacity=C)
        x64 = x.astype(np.float64)
        h = x64 @ w_r.astype(np.float64).T + bias.astype(np.float64)
        p = scipy.special.softmax(h, axis=1)
        order = np.argsort(-h, axis=1, kind="stable")[:, :2]
        slot, _, _ = _top2_priority_definition(order[:, 0].tolist(), order[:, 1].tolist(), N, C)
        every = np.stack([np.maximum(x64 @ w_in[i].astype(np.float64).T, 0) @ w_out[i].astype(np.float64).T
                          for i in range(N)])
        y = np.zeros((T, d))
        for t in range(T):
            for c in range(2):
                if slot[t, c] >= 0:
                    e = order[t, c]
                    y[t] += p[t, e] * every[e, t]
        assert np.array_equal(r["expert"], order)
        assert np.array_equal(r["slot"], slot)
        assert np.allclose(r["y"], y, rtol=1e-12, atol=1e-13), np.abs(r["y"] - y).max()
        f = np.bincount(order[:, 0], minlength=N) / T
        assert abs(r["aux"] - N * np.dot(f, p.mean(axis=0))) < 1e-12


def pin_top2_two_experts_dense_mixture(o):
    # N = 2 and C = T: every token uses both experts and nothing is dropped, so
    # the layer is the full softmax mixture p_0 E_0(x) + p_1 E_1(x) (closed form).
    rng = np.random.default_rng(22)
    T, d, F = 24, 6, 9
    x, w_r, bias, w_in, w_out = _random_problem(rng, T, d, F, 2)
    r = o.layer_fwd_top2(x, w_r, w_in, w_out, bias=bias, capacity=T)
    x64 = x.astype(np.float64)
    p = scipy.special.softmax(x64 @ w_r.astype(np.float64).T + bias.astype(np.float64), axis=1)
    mix = sum(p[:, [i]] * (np.maximum(x64 @ w_in[i].astype(np.float64).T, 0) @ w_out[i].astype(np.float64).T)
              for i in range(2))
    assert np.all(r["slot"] >= 0)
    assert r["counts"].tolist() == [T, T]
    assert np.allclose(r["y"], mix, rtol=1e-12, atol=1e-13)
    assert np.all(np.isinf(r["margin"][:, 1]))


def pin_top2_invariants(o):
    rng = np.random.default_rng(23)
    T, d, F, N = 300, 12, 20, 7
    x, w_r, bias, w_in, w_out = _random_problem(rng, T, d, F, N)
    r = o.layer_fwd_top2(x, w_r, w_in, w_out, bias=bias, capacity_factor=1.5, want_probs=True)
    C = r["capacity"]
    assert C == 65
    assert int(r["counts"].sum()) == 2 * T and int(r["counts_first"].sum()) == T
    assert np.all(r["expert"][:, 0] != r["expert"][:, 1])
    assert np.all(r["gate"][:, 0] >= r["gate"][:, 1]) and np.all(r["gate"].sum(axis=1) <= 1.0 + 1e-15)
    assert np.all(r["margin"] >= 0)
    kept = np.minimum(r["counts"], C)
    for e in range(N):
        mask = (r["expert"] == e) & (r["slot"] >= 0)
        assert int(mask.sum()) == kept[e]
        assert sorted(r["slot"][mask].tolist()) == list(range(kept[e]))
        for t, c in zip(*np.nonzero(mask)):
            assert r["slot_token"][e][r["slot"][t, c]] == t
        assert np.all(r["slot_token"][e][kept[e]:] == -1)
    both_dropped = (r["slot"] < 0).all(axis=1)
    assert np.all(r["y"][both_dropped] == 0.0)


# --------------------------------------------------------------------------
# Router statistics (the monitoring list)
# --------------------------------------------------------------------------

def pin_router_stats_16tok(o):
    # The 16-token example: counts [7, 4, 3, 2] at capacity 4 drop 3 of 16 tokens, keep 13 of the
    # 16 slots, and the busiest expert carries 7 / (16 / 4) = 1.75 times the uniform load.
    g = golden("overflow_16tok.json")
    counts = np.array(g["counts"], dtype=np.int32)
    T, N = int(counts.sum()), len(counts)
    st = o.router_stats(np.full((T, N), 1.0 / N), counts, g["capacity"])
    assert st["drop_fraction"] == 3 / 16 and st["capacity_utilisation"] == 13 / 16
    assert st["max_load"] == 1.75
    assert abs(st["entropy"] - np.log(N)) < 1e-15  # uniform probabilities: ln N


def pin_router_stats_entropy(o):
    # Entropy against scipy's (natural log), one-hot rows give 0, and the statistics of a routed batch.
    rng = np.random.default_rng(41)
    p = scipy.special.softmax(rng.standard_normal((50, 6)) * 2, axis=1)
    p[:3] = 0.0
    p[0, 2] = p[1, 0] = p[2, 5] = 1.0
    counts = np.array([20, 10, 9, 6, 3, 2], dtype=np.int32)
    st = o.router_stats(p, counts, 8)
    ref = scipy.stats.entropy(p, axis=1)
    assert np.all(ref[:3] == 0.0)
    assert abs(st["entropy"] - ref.mean()) < 1e-14
    assert st["drop_fraction"] == (12 + 2 + 1) / 50
    assert st["capacity_utilisation"] == (8 + 8 + 8 + 6 + 3 + 2) / 48
    assert st["max_load"] == 20 * 6 / 50
    assert o.router_stats(np.zeros((0, 6)), np.zeros(6, np.int32), 8)["entropy"] == 0.0


# --------------------------------------------------------------------------
# Backward pass (gradients of sum(y * dy) + g_aux * aux)
# --------------------------------------------------------------------------

def _layer_loss(o, x, w_r, bias, w_in, w_out, C, dy, g_aux):
    r = o.layer_fwd(x, w_r, w_in, w_out, bias=bias, capacity=C)
    return float(np.sum(r["y"] * dy) + g_aux * r["aux"]), r["expert"], r["slot"]


def _stable_problem(T, d, F, N, C, seed0):
    """A float32 problem whose routing and ReLU pattern survive small perturbations:
    top-2 logit margins >= 0.05 and |pre-activation| >= 0.05 on every kept token."""
    for seed in range(seed0, seed0 + 500):
        rng = np.random.default_rng(seed)
        x, w_r, bias, w_in, w_out = _random_problem(rng, T, d, F, N)
        w_r *= 3.0
        x64 = x.astype(np.float64)
        h = x64 @ w_r.astype(np.float64).T + bias
        srt = np.sort(h, axis=1)
        if N > 1 and (srt[:, -1] - srt[:, -2]).min() < 0.05:
            continue
        ids = np.argmax(h, axis=1)
        z = np.einsum("tk,tjk->tj", x64, w_in[ids].astype(np.float64))
        if np.abs(z).min() < 0.05:
            continue
        counts = np.bincount(ids, minlength=N)
        if N > 1 and (counts <= C).all():
            continue  # want some dropped tokens
        return x, w_r, bias, w_in, w_out
    raise AssertionError("no stable problem found")


def pin_bwd_finite_differences(o):
    # Central differences of the forward oracle's loss, one float32 element at a
    # time (the perturbation is the exact float32 step taken); routing and the
    # ReLU pattern stay fixed under the step, so the loss is smooth there.
    T, d, F, N, C = 7, 4, 5, 3, 2
    x, w_r, bias, w_in, w_out = _stable_problem(T, d, F, N, C, 300)
    rng = np.random.default_rng(31)
    dy = rng.standard_normal((T, d))
    g_aux = 0.7
    g = o.layer_bwd(x, w_r, w_in, w_out, dy, g_aux, bias=bias, capacity=C)
    _, ids0, slot0 = _layer_loss(o, x, w_r, bias, w_in, w_out, C, dy, g_aux)
    assert (slot0 < 0).any() and (slot0 >= 0).any()
    params = {"x": (x, "dx"), "w_r": (w_r, "dw_r"), "bias": (bias, "dbias"), "w_in": (w_in, "dw_in"),
              "w_out": (w_out, "dw_out")}
    for name, (arr, gname) in params.items():
        flat = arr.reshape(-1)
        num = np.zeros(flat.size)
        for i in range(flat.size):
            v = flat[i]
            steps = []
            for sgn in (1.0, -1.0):
                flat[i] = np.float32(v + sgn * np.float32(2.0 ** -11) * max(1.0, abs(float(v))))
                steps.append((float(flat[i]) - float(v),
                              _layer_loss(o, x, w_r, bias, w_in, w_out, C, dy, g_aux)))
                flat[i] = v
            (dp, (lp, ip, sp)), (dm, (lm, im, sm_)) = steps
            assert np.array_equal(ip, ids0) and np.array_equal(im, ids0), (name, i)
            assert np.array_equal(sp, slot0) and np.array_equal(sm_, slot0), (name, i)
            num[i] = (lp - lm) / (dp - dm)
        ana = g[gname].reshape(-1)
        scale = max(1.0, float(np.abs(ana).max()))
        assert np.allclose(num, ana, rtol=2e-5, atol=2e-5 * scale), (name, np.abs(num - ana).max())


def pin_bwd_matches_torch_autograd(o):
    # A dense formulation in torch (every expert on every token, masks from the
    # argmax and the first-C rule, gate = selected probability, f held constant),
    # differentiated by torch.autograd in float64.
    import torch
    for seed, (T, d, F, N, C, g_aux) in enumerate([(40, 8, 12, 4, 8, 0.3), (25, 6, 10, 3, 25, 0.0),
                                                   (30, 5, 7, 5, 3, 1.5)]):
        rng = np.random.default_rng(140 + seed)
        x, w_r, bias, w_in, w_out = _random_problem(rng, T, d, F, N)
        dy = rng.standard_normal((T, d))
        g = o.layer_bwd(x, w_r, w_in, w_out, dy, g_aux, bias=bias, capacity=C)
        tx, twr, tb = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (x, w_r, bias))
        twi, two = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (w_in, w_out))
        h = tx @ twr.T + tb
        p = torch.softmax(h, dim=1)
        ids = torch.argmax(h, dim=1)
        keep = torch.zeros(T, dtype=torch.float64)
        seen = [0] * N
        for t in range(T):
            e = int(ids[t])
            keep[t] = 1.0 if seen[e] < C else 0.0
            seen[e] += 1
        z = torch.einsum("tk,ejk->etj", tx, twi)
        out = torch.einsum("etj,ekj->etk", torch.relu(z), two)
        o_sel = out[ids, torch.arange(T)]
        gate = p[torch.arange(T), ids]
        y = keep[:, None] * gate[:, None] * o_sel
        f = torch.tensor(np.bincount(ids.numpy(), minlength=N) / T, dtype=torch.float64)
        aux = N * torch.sum(f * p.mean(dim=0))
        loss = torch.sum(y * torch.tensor(dy)) + g_aux * aux
        loss.backward()
        for name, tg in (("dx", tx), ("dw_r", twr), ("dbias", tb), ("dw_in", twi), ("dw_out", two)):
            assert np.allclose(g[name], tg.grad.numpy(), rtol=1e-11, atol=1e-12), (name, seed)


def pin_bwd_single_expert(o):
    # N = 1: p = 1 identically, so the router gets no gradient (even from aux),
    # and dx is the dense FFN's backward (numpy closed form).
    rng = np.random.default_rng(32)
    T, d, F = 12, 6, 9
    x, w_r, bias, w_in, w_out = _random_problem(rng, T, d, F, 1)
    dy = rng.standard_normal((T, d))
    g = o.layer_bwd(x, w_r, w_in, w_out, dy, 2.0, bias=bias, capacity=T)
    assert np.all(g["dw_r"] == 0.0) and np.all(g["dbias"] == 0.0)
    x64, wi, wo = x.astype(np.float64), w_in[0].astype(np.float64), w_out[0].astype(np.float64)
    z = x64 @ wi.T
    du = dy @ wo
    dz = du * (z > 0)
    assert np.allclose(g["dx"], dz @ wi, rtol=1e-12, atol=1e-13)
    assert np.allclose(g["dw_out"][0], dy.T @ np.maximum(z, 0), rtol=1e-12, atol=1e-13)
    assert np.allclose(g["dw_in"][0], dz.T @ x64, rtol=1e-12, atol=1e-13)


def pin_bwd_aux_only_and_dropped(o):
    # dy = 0: the expert weights get no gradient and the router gradient is the
    # aux term alone, dh_i = p_i (c_i - sum_j p_j c_j) with c_i = g_aux N f_i / T.
    # With g_aux = 0 a dropped token gets no gradient at all.
    rng = np.random.default_rng(33)
    T, d, F, N, C = 30, 6, 8, 4, 5
    x, w_r, bias, w_in, w_out = _random_problem(rng, T, d, F, N)
    g = o.layer_bwd(x, w_r, w_in, w_out, np.zeros((T, d)), 1.3, bias=bias, capacity=C)
    assert np.all(g["dw_in"] == 0.0) and np.all(g["dw_out"] == 0.0)
    x64 = x.astype(np.float64)
    h = x64 @ w_r.astype(np.float64).T + bias
    p = scipy.special.softmax(h, axis=1)
    f = np.bincount(np.argmax(h, axis=1), minlength=N) / T
    c = 1.3 * N * f / T
    dh = p * (c - (p * c).sum(axis=1, keepdims=True))
    assert np.allclose(g["dw_r"], dh.T @ x64, rtol=1e-12, atol=1e-14)
    assert np.allclose(g["dbias"], dh.sum(axis=0), rtol=1e-12, atol=1e-14)
    assert np.allclose(g["dx"], dh @ w_r.astype(np.float64), rtol=1e-12, atol=1e-14)
    dy = rng.standard_normal((T, d))
    g0 = o.layer_bwd(x, w_r, w_in, w_out, dy, 0.0, bias=bias, capacity=C)
    slot = o.route(x, w_r, bias, capacity=C)["slot"]
    assert (slot < 0).any()
    assert np.all(g0["dx"][slot < 0] == 0.0)


PINS = {name: fn for name, fn in sorted(globals().items()) if name.startswith("pin_") and callable(fn)}
