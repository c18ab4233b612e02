"""Plant plausible mistakes in copies of the oracle and check that the pins catch each.

Each mutant is a textual edit of ``oracle/switch_oracle.c`` (the original is
never touched), compiled with gcc into a temporary shared object and run
through every pin in ``oracle_pins.py``.  A mutant that no pin rejects means
the pins leave that part of the oracle unchecked.  Every edit keeps memory
accesses in bounds, so a mutant can give wrong answers but cannot crash.
"""
from pathlib import Path

import pytest

import oracle
from oracle_pins import PINS

SRC = Path(oracle.__file__).resolve().parent / "switch_oracle.c"

MUTANTS = {
    # router: transposed W_r operand (k < d, i < N keeps k*N+i < N*d)
    "router_transposed_weight": ("(double)w_r[(int64_t)i * d + k]", "(double)w_r[(int64_t)k * N + i]"),
    "router_bias_dropped": ("acc += (double)bias[i];", "acc += 0.0;"),
    "router_bias_sign": ("acc += (double)bias[i];", "acc -= (double)bias[i];"),
    # top-1: ties resolved to the highest index instead of the lowest
    "argmax_last_on_ties": ("if (row[i] > m) {", "if (row[i] >= m) {"),
    # softmax: numerator not shifted by the row maximum while the denominator is
    "softmax_unshifted_numerator": ("p[t * (int64_t)N + i] = exp(row[i] - m) / denom;",
                                    "p[t * (int64_t)N + i] = exp(row[i]) / denom;"),
    "softmax_denominator_missing_term": ("for (int32_t i = 0; i < N; ++i)\n            denom += exp(row[i] - m);",
                                         "for (int32_t i = 1; i < N; ++i)\n            denom += exp(row[i] - m);"),
    "gate_is_first_prob": ("gate[t] = p[t * (int64_t)N + arg];", "gate[t] = p[t * (int64_t)N + 0];"),
    # capacity: floor instead of ceil, or no rounding snap
    "capacity_floor": ("double cap = fabs(exact - nearest) <= 1e-9 ? nearest : ceil(exact);",
                       "double cap = floor(exact);"),
    "capacity_off_by_one": ("double cap = fabs(exact - nearest) <= 1e-9 ? nearest : ceil(exact);",
                            "double cap = (fabs(exact - nearest) <= 1e-9 ? nearest : ceil(exact)) + 1.0;"),
    # assignment: slot numbering starts at 1; keeps C+... ; reverse token order
    "slot_one_based": ("slot[t] = position;", "slot[t] = position + 1;"),
    "assign_reverse_order": ("for (int64_t t = 0; t < T; ++t) {\n        int32_t e = expert[t];",
                             "for (int64_t t = T - 1; t >= 0; --t) {\n        int32_t e = expert[t];"),
    # aux: N factor dropped; f and P not normalised by T
    "aux_missing_N": ("return (double)N * total;", "return total;"),
    "aux_P_not_averaged": ("double P = prob_sum[i] / (double)T;", "double P = prob_sum[i];"),
    # expert FFN: ReLU dropped, wrong activation side, transposed W_out, gate not applied
    "ffn_no_relu": ("u[j] = acc > 0.0 ? acc : 0.0;", "u[j] = acc;"),
    "ffn_relu_inverted": ("u[j] = acc > 0.0 ? acc : 0.0;", "u[j] = acc < 0.0 ? acc : 0.0;"),
    "ffn_w_out_transposed": ("load_elem(w_out, w_dtype, (int64_t)k * F + j)", "load_elem(w_out, w_dtype, (int64_t)j * d + k)"),
    "ffn_w_in_transposed": ("load_elem(w_in, w_dtype, (int64_t)j * d + k)", "load_elem(w_in, w_dtype, (int64_t)k * F + j)"),
    "ffn_gate_missing": ("y_row[k] = gate * acc;", "y_row[k] = acc;"),
    "dropped_token_not_zeroed": ("if (slot[t] < 0) {", "if (slot[t] < -1) {"),
    # top-2: second choice on ties goes to the highest index; may repeat the first choice
    "top2_second_ties_last": ("if (i != first && (second < 0 || row[i] > row[second]))",
                              "if (i != first && (second < 0 || row[i] >= row[second]))"),
    "top2_second_may_be_first": ("if (i != first && (second < 0 || row[i] > row[second]))",
                                 "if ((second < 0 || row[i] > row[second]))"),
    # top-2 gates renormalised over the selected pair
    "top2_gate_renormalised": ("gate2[2 * t] = p[t * (int64_t)N + first];",
                               "gate2[2 * t] = p[t * (int64_t)N + first] / (p[t * (int64_t)N + first] + "
                               "p[t * (int64_t)N + second]);"),
    "top2_margin_second_wrong": ("margin2[2 * t + 1] = (N == 2) ? INFINITY : row[second] - third;",
                                 "margin2[2 * t + 1] = (N == 2) ? INFINITY : row[first] - third;"),
    "top2_softmax_denominator_missing_term": ("for (int32_t j = 0; j < N; ++j)\n            denom += exp(row[j] - m);",
                                              "for (int32_t j = 1; j < N; ++j)\n            denom += exp(row[j] - m);"),
    # top-2 capacity: token-major priority instead of first choices first
    "top2_token_major_priority": ("for (int c = 0; c < 2; ++c) {\n        for (int64_t t = 0; t < T; ++t) {",
                                  "for (int64_t t = 0; t < T; ++t) {\n        for (int c = 0; c < 2; ++c) {"),
    # aux fed with the counts of both choices
    "top2_first_counts_both_choices": ("if (c == 0)\n                counts_first[e] += 1;",
                                       "counts_first[e] += 1;"),
    # top-2 output: second choice never added
    "top2_output_first_only": ("for (int c = 0; c < 2; ++c) {\n            if (slot2[2 * t + c] < 0)",
                               "for (int c = 0; c < 1; ++c) {\n            if (slot2[2 * t + c] < 0)"),
    # backward: ReLU mask dropped; gate missing from the expert-output gradient
    "bwd_relu_mask_dropped": ("dz[j] = z[j] > 0.0 ? acc : 0.0;", "dz[j] = acc;"),
    "bwd_forward_relu_dropped": ("u[j] = z[j] > 0.0 ? z[j] : 0.0;", "u[j] = z[j];"),
    "bwd_gate_missing": ("dout[k] = gate[t] * dy[t * (int64_t)d + k];", "dout[k] = dy[t * (int64_t)d + k];"),
    # softmax backward with the wrong sign of the centring term
    "bwd_softmax_sign": ("dht[i] = pt[i] * (dht[i] - dot);", "dht[i] = pt[i] * (dht[i] + dot);"),
    "bwd_aux_missing_N": ("double dp = g_aux * (double)N * ((double)counts[i] / (double)T) / (double)T;",
                          "double dp = g_aux * ((double)counts[i] / (double)T) / (double)T;"),
    # dropped tokens still back-propagate through the expert
    "bwd_dropped_tokens_pass": ("if (expert[t] != e || slot[t] < 0)\n                continue;",
                                "if (expert[t] != e)\n                continue;"),
    "bwd_dw_out_transposed": ("dwout_e[(int64_t)k * F + j] += dout[k] * u[j];",
                              "dwout_e[(int64_t)j * d + k] += dout[k] * u[j];"),
    "bwd_router_dx_transposed_weight": ("router_part += dht[i] * w_r[(int64_t)i * d + k];",
                                        "router_part += dht[i] * w_r[(int64_t)k * N + i];"),
    "bwd_router_dx_missing": ("dx[t * (int64_t)d + k] += router_part;", "dx[t * (int64_t)d + k] += 0.0 * router_part;"),
    "bwd_gate_grad_uses_dy_only": ("gg += dy[t * (int64_t)d + k] * acc;", "gg += dy[t * (int64_t)d + k];"),
    # router statistics: log base 2; overflow counted on every token; utilisation over T
    "stats_entropy_log2": ("h -= p * log(p);", "h -= p * log2(p);"),
    "stats_drop_no_clamp": ("dropped += c > C ? c - C : 0;", "dropped += c - C;"),
    "stats_utilisation_over_T": ("out[2] = (double)kept / ((double)N * (double)C);",
                                 "out[2] = (double)kept / (double)T;"),
    # bf16 loads: wrong half of the 32-bit pattern
    "bf16_wrong_shift": ("uint32_t wide = (uint32_t)bits << 16;", "uint32_t wide = (uint32_t)bits << 15;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    text = SRC.read_text()
    assert text.count(old) == 1, f"mutation site for {name} not found exactly once"
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new))
    so = oracle.build(force=True, source=src, out=tmp_path / f"lib_{name}.so")
    mutant = oracle.Oracle(oracle.load(so))
    failed = []
    for pin_name, pin in PINS.items():
        try:
            pin(mutant)
        except AssertionError:
            failed.append(pin_name)
    assert failed, f"no pin rejects mutant {name}"
