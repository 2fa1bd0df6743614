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
    "router_weight_transposed": ("(double)w_router[(size_t)e * d + i]", "(double)w_router[(size_t)i * E + e]"),
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
    "gate_up_rows_swapped": ("const uint16_t* gr = wgu + (size_t)n * d;\n        const uint16_t* ur = wgu + (size_t)(f + n) * d;",
                             "const uint16_t* gr = wgu + (size_t)(f + n) * d;\n        const uint16_t* ur = wgu + (size_t)n * d;"),
    "gate_up_interleaved": ("const uint16_t* gr = wgu + (size_t)n * d;\n        const uint16_t* ur = wgu + (size_t)(f + n) * d;",
                            "const uint16_t* gr = wgu + (size_t)(2 * n) * d;\n        const uint16_t* ur = wgu + (size_t)(2 * n + 1) * d;"),
    "down_transposed": ("s += h[n] * bf16_to_double(dr[n]);", "s += h[n] * bf16_to_double(wd[(size_t)n * d + c]);"),
    "routing_weight_dropped": ("acc[c] += scale * s;", "acc[c] += s;"),
    "last_expert_dropped": ("for (int j = 0; j < J->k; ++j) {", "for (int j = 0; j < J->k - 1; ++j) {"),
    "shared_expert_half_weight": ("J->wd_s, 1.0, h, acc)", "J->wd_s, 0.5, h, acc)"),
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
