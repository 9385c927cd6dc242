"""Plant one mistake at a time in a private copy of the oracle (CPU only) and
require that at least one pin catches it.  This is how we know the pins are
sharp enough to trust the oracle."""
import os

import pytest

import oracle
from oracle_checks import ALL_CHECKS

SRC = os.path.join(os.path.dirname(oracle.__file__), "moe_oracle.c")

MUTANTS = {
    "silu_sign": [("z / (1.0 + exp(-z))", "z / (1.0 + exp(z))")],
    "swap_w1_w3": [("a[f] += xj * elem(w1,", "a[f] += xj * elem(@W3@,"),
                   ("b[f] += xj * elem(w3,", "b[f] += xj * elem(w1,"),
                   ("@W3@", "w3")],
    "silu_on_up_proj": [("a[f] = oracle_silu(a[f]) * b[f];", "a[f] = a[f] * oracle_silu(b[f]);")],
    "tie_break_high_index": [("L[e] > L[best]", "L[e] >= L[best]")],
    "gate_dropped": [("yt[i] += g * o[i];", "yt[i] += o[i];")],
    "gate_unnormalised": [("gate[k] = exp(L[idx[k]] - m) / z;", "gate[k] = exp(L[idx[k]] - m);")],
    "router_transposed": [("(size_t)j * n + e", "(size_t)e * d + j")],
    "w2_transposed": [("out[i] += a[f] * elem(w2, w_dt, row + i);",
                       "out[i] += a[f] * elem(w2, w_dt, ebase2 + (size_t)i * F + f);")],
    "bf16_shift": [("<< 16;", "<< 15;")],
    "dispatch_slot_major": [("        for (int64_t t = 0; t < T; ++t)\n            for (int k = 0; k < K; ++k)\n                if (idx[t * K + k] == e) {",
                             "        for (int k = 0; k < K; ++k)\n            for (int64_t t = 0; t < T; ++t)\n                if (idx[t * K + k] == e) {")],
    "softmax_first_logit_only": [("z += exp(L[idx[k]] - m);", "z += (k == 0) ? 1.0 : 0.0;")],
    "stats_f_over_tokens": [("f[e] /= (double)(T * K);", "f[e] /= (double)T;")],
    "stats_P_unnormalised": [("P[e] += exp(L[e] - m) / z;", "P[e] += exp(L[e] - m);")],
    "expert_choice_lowest_scores": [("    if (sa > sb) return -1;\n    if (sa < sb) return 1;",
                                     "    if (sa < sb) return -1;\n    if (sa > sb) return 1;")],
    "expert_choice_ties_high_token": [("return (ta < tb) ? -1 : (ta > tb);", "return (ta > tb) ? -1 : (ta < tb);")],
    "expert_choice_gate_unnormalised": [("S[t * n + e] = exp(S[t * n + e] - m) / z;", "S[t * n + e] = exp(S[t * n + e] - m);")],
    "e4m3_ties_up": [("return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;", "return f + 1.0;")],
    "e4m3_no_act_scale": [("double av = a[f] * sx * s1[(size_t)e * F + f];", "double av = a[f] * s1[(size_t)e * F + f];")],
    "e4m3_no_down_scale": [("yt[i] += g * o * sh * s2[(size_t)e * d + i];", "yt[i] += g * o * s2[(size_t)e * d + i];")],
    "e2m1_ties_up": [("q = 0.5 * round_half_even(a / 0.5);", "q = 0.5 * floor(a / 0.5 + 0.5);")],
    "e2m1_bias_0": [("ldexp(1.0 + 0.5 * m, e - 1)", "ldexp(1.0 + 0.5 * m, e)")],
    "fp4_tensor_scale_448": [("amax / 2688.0f", "amax / 448.0f")],
    "fp4_nibbles_swapped": [("(uint8_t)(code << (4 * h))", "(uint8_t)(code << (4 * (1 - h)))")],
    "fp4_block_scale_no_div6": [("float qb = (amax_b / 6.0f) / st;", "float qb = amax_b / st;")],
    "w4a4_no_row_scale": [("return fp4_lut[code] * e4m3_lut[bscale[j / 16]] * (double)rs;",
                           "return fp4_lut[code] * e4m3_lut[bscale[j / 16]];")],
    "w4a4_silu_on_up_proj": [("hf[f] = round_bf16((float)(oracle_silu(a[f]) * b[f]));",
                              "hf[f] = round_bf16((float)(a[f] * oracle_silu(b[f])));")],
    "fp4_rows_block_scale_no_div6": [("int sb_code = oracle_e4m3_encode((double)((amax_b / 6.0f) / rs));",
                                      "int sb_code = oracle_e4m3_encode((double)(amax_b / rs));")],
    "e4m3_scale_over_256": [("amax / 448.0f", "amax / 256.0f")],
    "e4m3_bias_8": [("v = ldexp(1.0 + m / 8.0, e - 7);", "v = ldexp(1.0 + m / 8.0, e - 8);")],
    "gates_bf16_truncate": [("if (low > 0x8000u || (low == 0x8000u && (hi & 1u)))", "if (0)")],
    "gates_bf16_ties_up": [("if (low > 0x8000u || (low == 0x8000u && (hi & 1u)))", "if (low >= 0x8000u)")],
    # straight from double to bf16: the bits lost in the fp32 step break a bf16 tie
    "gates_bf16_no_fp32_step": [("if (low > 0x8000u || (low == 0x8000u && (hi & 1u)))",
                                 "if (low > 0x8000u || (low == 0x8000u && ((hi & 1u) || (double)f < gate[i])))")],
    "capacity_keeps_one_more": [("if (row - offsets[e] < capacity) {", "if (row - offsets[e] <= capacity) {")],
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    src = open(SRC).read()
    for old, new in MUTANTS[name]:
        assert old in src, "mutation anchor not found: %r" % old
        src = src.replace(old, new)
    path = tmp_path / "mutant.c"
    path.write_text(src)
    so = oracle.compile_source(str(path), str(tmp_path / ("libmutant_%s.so" % name)))
    O = oracle.Oracle(so)
    caught = []
    for check in ALL_CHECKS:
        try:
            check(O)
        except (AssertionError, ValueError):
            caught.append(check.__name__)
    assert caught, "no pin caught mutant %s" % name
