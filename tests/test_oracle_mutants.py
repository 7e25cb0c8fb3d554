"""Plant plausible mistakes in a COPY of the oracle and show the pins catch each.

The committed oracle is never modified: each mutant is a textual edit of
oracle.c compiled to a temporary library on the CPU.
"""
import os

import pytest

import oracle
import pins

ORACLE_C = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (name, text in oracle.c, replacement).  Each is a mistake a careful reader
# could plausibly make, and each keeps every index in range so that the
# mutant cannot corrupt memory: a flipped tie-break, a dropped bias, weights
# normalised over all experts, an unstable order inside an expert, gate and
# up swapped, a wrong SiLU sign, a transposed down-projection weight, an
# unweighted combine, capacity slots filled in reverse, a reversed overflow
# segment, logits accumulated in fp32; for the fp8 variant a wrong exponent
# bias, ties rounded away from zero, subnormals flushed to zero, a scale one
# binade too high and weight codes left in the untransposed layout.
MUTANTS = [
    ("tie_break_highest_index", "    return i < j;\n}", "    return i > j;\n}"),
    ("bias_dropped", "if (bias) l = l + bias[e];", "(void)bias;"),
    ("softmax_over_all_experts",
     "        for (int j = 0; j < k; ++j) w[(size_t)t * k + j] = (float)(ex[j] / s);",
     "        for (int e = 0; e < E; ++e) if (!taken[e]) s += exp((double)l[e] - m);\n"
     "        for (int j = 0; j < k; ++j) w[(size_t)t * k + j] = (float)(ex[j] / s);"),
    ("unstable_order_within_expert", "row = (int64_t)offsets[e] + r;", "row = (int64_t)offsets[e + 1] - 1 - r;"),
    ("gate_up_swapped",
     "const double silu = g[f] / (1.0 + exp(-g[f]));\n        hrow[f] = double_to_bf16(silu * u[f]);",
     "const double silu = u[f] / (1.0 + exp(-u[f]));\n        hrow[f] = double_to_bf16(silu * g[f]);"),
    ("silu_sign", "g[f] / (1.0 + exp(-g[f]))", "g[f] / (1.0 + exp(g[f]))"),
    ("down_transposed",
     "const uint16_t *wd = wd_e + (size_t)f * H;\n        for (int c = 0; c < H; ++c) y[c] += hv * bf16_to_double(wd[c]);",
     "for (int c = 0; c < H; ++c) y[c] += hv * bf16_to_double(wd_e[((size_t)c * F + f) % ((size_t)F * H)]);"),
    ("combine_unweighted",
     "const float prod = w[(size_t)t * k + j] * (float)bf16_to_double(y[(size_t)r * H + c]);",
     "const float prod = (float)bf16_to_double(y[(size_t)r * H + c]);"),
    ("capacity_slots_reversed", "row = (int64_t)e * C + r;", "row = (int64_t)e * C + (C - 1 - r);"),
    ("overflow_reversed", "row = (int64_t)E * C + spill_off[e] + (r - C);",
     "row = (int64_t)E * C + spill_off[e + 1] - 1 - (r - C);"),
    ("e4m3_exponent_bias_8", "ldexp(1.0 + man / 8.0, ex - 7)", "ldexp(1.0 + man / 8.0, ex - 8)"),
    ("e4m3_ties_away_from_zero", "double r = nearbyint(ldexp(a, 3 - e));", "double r = round(ldexp(a, 3 - e));"),
    ("e4m3_subnormals_flushed", "code = (uint8_t)r; /* r == 8", "code = (uint8_t)(r >= 8.0 ? r : 0.0); /* r == 8"),
    ("fp8_scale_one_binade_high", "return (float)ldexp(1.0, c - 8);", "return (float)ldexp(1.0, c - 7);"),
    ("fp8_weights_not_transposed", "q + ((size_t)e * N + n) * K, 1);", "q + (size_t)e * K * N + n, N);"),
    ("logit_accumulated_in_float",
     "            double s = 0.0;\n            for (int h = 0; h < H; ++h) s += bf16_to_double",
     "            float s = 0.0f;\n            for (int h = 0; h < H; ++h) s += (float)bf16_to_double"),
]


def _mutant_oracle(tmp_path, name, old, new):
    src = open(ORACLE_C).read()
    assert src.count(old) == 1, "mutation anchor for %s must occur exactly once" % name
    path = tmp_path / ("oracle_%s.c" % name)
    path.write_text(src.replace(old, new))
    so = oracle.build(force=True, src=str(path), out=str(tmp_path / ("oracle_%s.so" % name)))
    return oracle.Oracle(oracle.load(so))


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    orc = _mutant_oracle(tmp_path, name, old, new)
    caught = []
    for check in pins.ALL_CHECKS:
        try:
            check(orc)
        except (AssertionError, ValueError, IndexError):
            caught.append(check.__name__)
    assert caught, "no pin caught mutant %s" % name
