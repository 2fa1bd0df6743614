"""Plant plausible mistakes in copies of the oracle (on the CPU) and check that the pins catch each one.

This shows the pins constrain every part of the oracle: a dropped term, a wrong sign, a swapped or
transposed operand, a broken tie rule or an unstable grouping each fails at least one pin.
"""
import os

import pytest

import oracle
from oracle_pins import PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "moe_oracle.c")

MUTATIONS = {
    "router_bias_dropped": ("if (bias) s += (double)bias[e];", ""),
    "router_weight_transposed": ("s += bf16_to_double(x[(size_t)t * d + i]) * (double)w_router[(size_t)e * d + i]",
                                 "s += bf16_to_double(x[(size_t)t * d + i]) * (double)w_router[(size_t)i * E + e]"),
    "topk_tie_prefers_higher_id": ("l[e] > l[best]", "l[e] >= l[best]"),
    "softmax_missing_normalisation": ("for (int j = 0; j < k; ++j) wt[j] /= z;\n        } else if",
                                      "\n        } else if"),
    "renorm_not_renormalised": ("for (int j = 0; j < k; ++j) wt[j] /= zsel;", ""),
    "sigmoid_sign_flipped": ("1.0 / (1.0 + exp(-(double)l[it[j]]))", "1.0 / (1.0 + exp((double)l[it[j]]))"),
    "margin_wrong_rank": ("margin[t] = v[k - 1] - v[k];", "margin[t] = v[0] - v[k];"),
    "permute_slot_not_token": ("perm_src[r] = (int32_t)(a / k);", "perm_src[r] = (int32_t)(a % k);"),
    "permute_offsets_inclusive": ("offsets[e + 1] = offsets[e] + counts[e];",
                                  "offsets[e + 1] = offsets[e] + counts[e] + (e == 0);"),
    "permute_unstable": ("for (long a = 0; a < R; ++a) {\n        int32_t r",
                         "for (long a = R - 1; a >= 0; --a) {\n        int32_t r"),
    "silu_sign_flipped": ("h[n] = g / (1.0 + exp(-g)) * u;", "h[n] = g / (1.0 + exp(g)) * u;"),
    "silu_on_up_not_gate": ("h[n] = g / (1.0 + exp(-g)) * u;", "h[n] = u / (1.0 + exp(-u)) * g;"),
    # the forward loop's gate/up rows (the anchor runs into its accumulator declaration, which is unique)
    "gate_up_rows_swapped": ("const uint16_t* gr = wgu + (size_t)n * d;\n        const uint16_t* ur = wgu + (size_t)(f + n) * d;\n        double g = 0.0, u = 0.0;",
                             "const uint16_t* gr = wgu + (size_t)(f + n) * d;\n        const uint16_t* ur = wgu + (size_t)n * d;\n        double g = 0.0, u = 0.0;"),
    "gate_up_interleaved": ("const uint16_t* gr = wgu + (size_t)n * d;\n        const uint16_t* ur = wgu + (size_t)(f + n) * d;\n        double g = 0.0, u = 0.0;",
                            "const uint16_t* gr = wgu + (size_t)(2 * n) * d;\n        const uint16_t* ur = wgu + (size_t)(2 * n + 1) * d;\n        double g = 0.0, u = 0.0;"),
    "backward_gate_up_rows_swapped": ("const uint16_t* gr = wgu + (size_t)n * d;\n        const uint16_t* ur = wgu + (size_t)(f + n) * d;\n        double* dgr",
                                      "const uint16_t* gr = wgu + (size_t)(f + n) * d;\n        const uint16_t* ur = wgu + (size_t)n * d;\n        double* dgr"),
    "down_transposed": ("s += h[n] * bf16_to_double(dr[n]);", "s += h[n] * bf16_to_double(wd[(size_t)n * d + c]);"),
    "routing_weight_dropped": ("acc[c] += scale * s;", "acc[c] += s;"),
    "last_expert_dropped": ("for (int j = 0; j < J->k; ++j) {", "for (int j = 0; j < J->k - 1; ++j) {"),
    "shared_expert_half_weight": ("J->wd_s, 1.0, h, acc)", "J->wd_s, 0.5, h, acc)"),
    "e2m1_exponent_bias_dropped": ("ldexp(1.0 + 0.5 * m, e - 1)", "ldexp(1.0 + 0.5 * m, e)"),
    "e2m1_subnormal_as_one": ("e == 0 ? 0.5 * m :", "e == 0 ? 1.0 * m :"),
    "mxfp4_ties_to_lower_code": ("(dist == bestd && (c & 1) == 0 && (best & 1) == 1)", "0"),
    "mxfp4_ties_away_from_zero": ("(dist == bestd && (c & 1) == 0 && (best & 1) == 1)", "dist == bestd"),
    "mxfp4_scale_emax_off_by_one": ("shared = ex - 1 - 2;", "shared = ex - 1 - 1;"),
    "mxfp4_scale_ceil_not_floor": ("shared = ex - 1 - 2;", "shared = ex - 2;"),
    "mxfp4_sign_dropped": ("e2m1_nearest(p) | ((v[i] >> 15) ? 8 : 0)", "e2m1_nearest(p)"),
    "mxfp4_natural_nibble_order": (
        "word |= (uint32_t)code[8 * j + 2 * i] << (4 * i);\n                    word |= (uint32_t)code[8 * j + 2 * i + 1] << (16 + 4 * i);",
        "word |= (uint32_t)code[8 * j + 2 * i] << (8 * i);\n                    word |= (uint32_t)code[8 * j + 2 * i + 1] << (8 * i + 4);"),
    "mxfp4_scale_layout_row_major": ("s[((size_t)g * nb + b) * N + n] = (uint8_t)(shared + 127);",
                                     "s[((size_t)g * N + n) * nb + b] = (uint8_t)(shared + 127);"),
    "mxfp4_zero_block_scale_max": ("int shared = -127;", "int shared = 127;"),
    "mxfp4_decode_odd_even_swapped": ("const int nib = (e % 2 == 0) ? e / 2 : 4 + e / 2;",
                                      "const int nib = (e % 2 == 1) ? e / 2 : 4 + e / 2;"),
    "backward_silu_prime_missing_term": ("(s * (1.0 + g[n] * (1.0 - s)))", "s"),
    "backward_du_uses_gate": ("const double du = dh[n] * a;", "const double du = dh[n] * g[n];"),
    "backward_routing_weight_dropped": ("const double dyc = scale * dyt[c];", "const double dyc = dyt[c];"),
    "backward_dwd_transposed": ("dwd[(size_t)c * f + n] += dyc * h[n];", "dwd[(size_t)n * d + c] += dyc * h[n];"),
    "backward_dx_missing_up_path": ("dxt[i] += dg * bf16_to_double(gr[i]) + du * bf16_to_double(ur[i]);",
                                    "dxt[i] += dg * bf16_to_double(gr[i]);"),
    "backward_dw_scaled_by_w": ("*dwt = s;", "*dwt = scale * s;"),
    "backward_shared_expert_skipped": ("if (shared && !status)\n            swiglu_expert_backward(",
                                       "if (0)\n            swiglu_expert_backward("),
    "router_backward_softmax_not_centred": ("g = wt[j] * (dwt[j] - dot);", "g = wt[j] * dwt[j];"),
    "router_backward_sigmoid_derivative_dropped": ("g = s * (1.0 - s) / S * (dwt[j] - dot);", "g = s / S * (dwt[j] - dot);"),
    "router_backward_dx_uses_x": ("dx[(size_t)t * d + i] += g * (double)w_router[(size_t)e * d + i];",
                                  "dx[(size_t)t * d + i] += g * bf16_to_double(x[(size_t)t * d + i]);"),
    "grad_entries_routing_weight_dropped": ("for (int q = 0; q < n_entries; ++q) out[q] += wt * dyt[a[q]] * h[b[q]];",
                                            "for (int q = 0; q < n_entries; ++q) out[q] += dyt[a[q]] * h[b[q]];"),
    "grad_entries_up_uses_silu_prime": (": dh[n] * g[n] * sg;", ": dh[n] * u[n] * sg;"),
    "mxfp4_decode_scale_bias": ("oracle_e2m1_value(code) * ldexp(1.0, sc - 127)", "oracle_e2m1_value(code) * ldexp(1.0, sc - 126)"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    so = str(tmp_path / "mutant.so")
    oracle.build(force=True, src=str(mutated), out=so)
    lib = oracle.load(so)
    caught = []
    for pin in PINS:
        try:
            pin(lib)
        except Exception as exc:  # AssertionError or a ValueError raised by a broken routine
            caught.append((pin.__name__, type(exc).__name__))
    assert caught, f"no pin caught mutation {name}"
