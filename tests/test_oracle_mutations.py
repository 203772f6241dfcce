"""Plant plausible mistakes in a copy of the oracle and check that the pins catch each.

Each mutation edits one line of a temporary copy of ``oracle/bnb4_oracle.c``,
builds it on the CPU and runs the pin checks against it.  A mutation that no
pin notices would mean the pins do not cover that step.
"""
import ctypes
import os
import shutil
import subprocess
import tempfile

import pytest

import oracle
import test_oracle as pins  # noqa: E402  (tests/ is on sys.path under pytest)
import test_oracle_double_quant as dq_pins  # noqa: E402
import test_oracle_8bit as q8_pins  # noqa: E402
import test_oracle_embedding as emb_pins  # noqa: E402

SRC = os.path.join(os.path.dirname(oracle.__file__), "bnb4_oracle.c")

MUTATIONS = {
    "ties_to_largest_index": ("if (d < bd) {", "if (d <= bd) {"),
    "nibble_order_swapped": ("packed[i >> 1] |= (uint8_t)(idx << 4);\n            else\n                packed[i >> 1] |= (uint8_t)idx;",
                             "packed[i >> 1] |= (uint8_t)idx;\n            else\n                packed[i >> 1] |= (uint8_t)(idx << 4);"),
    "absmax_without_abs": ("float a = fabsf(load_elem(x, dtype, i));", "float a = load_elem(x, dtype, i);"),
    "reciprocal_instead_of_quotient": ("load_elem(x, dtype, i) / amax;", "load_elem(x, dtype, i) * (1.0f / amax);"),
    "zero_block_not_special": ("(amax == 0.0f) ? 0.0f : load_elem", "(0) ? 0.0f : load_elem"),
    "dequant_operands_rounded_to_bf16": (
        "float p = c * a;\n    return p;",
        "float p = oracle_bf16_to_f32(oracle_f32_to_bf16_rne(c)) *"
        " oracle_bf16_to_f32(oracle_f32_to_bf16_rne(a));\n    return p;"),
    "dequant_skips_fp32_rounding": (
        "store_elem(out, out_dtype, i, dequant_f32(packed, absmax, i, blocksize, code));",
        "if (out_dtype == ORACLE_BF16) ((uint16_t *)out)[i] = encode_format(round_to_format("
        "(double)code[code_index(packed, i)] * (double)absmax[i / blocksize], 8, -126,"
        " ldexp(2.0 - ldexp(1.0, -7), 127)), 7, 127, -126, 255);"
        " else store_elem(out, out_dtype, i, dequant_f32(packed, absmax, i, blocksize, code));"),
    "fp4_exponent_bias": ("(1.0 + 0.5 * m) * ldexp(1.0, e - 1)", "(1.0 + 0.5 * m) * ldexp(1.0, e)"),
    "nf4_literal_typo": ("-0.2844414f", "-0.2844441f"),
    "rounding_truncates": ("double r = nearbyint(a / quantum) * quantum;", "double r = floor(a / quantum) * quantum;"),
    "forward_weight_transposed": ("dequant_f32(packed, absmax, j * K + k, blocksize, code);\n        acc += xv * wv;",
                                  "dequant_f32(packed, absmax, k * N + j, blocksize, code);\n        acc += xv * wv;"),
    "forward_bias_dropped": ("acc += (double)load_elem(bias, x_dtype, j);", "acc += 0.0;"),
    "backward_weight_transposed": ("j * K + k, blocksize, code);\n        acc += g * wv;",
                                   "k * N + j, blocksize, code);\n        acc += g * wv;"),
    "double_quant_truncates": ("const float r = rintf(t);", "const float r = truncf(t);"),
    "double_quant_scale_is_first_value": ("if (absmax[i] > s)\n                s = absmax[i];",
                                          "if (i == g0)\n                s = absmax[i];"),
    "dequant_absmax_other_rounding_order": ("out[i] = (float)q[i] * step;",
                                            "out[i] = (float)q[i] * scales[i / group] / 255.0f;"),
    # the mistake the pages report: the normalised value snapped to a 65536-point grid
    "quantize_8bit_snaps_to_grid": ("q[i] = (uint8_t)nearest_code8(v, code);",
                                    "q[i] = (uint8_t)nearest_code8((float)(nearbyint(((double)v + 1.0) * 32767.5)"
                                    " / 32767.5 - 1.0), code);"),
    "quantize_8bit_ties_to_largest": ("if (dist_less(dist, best_d)) {", "if (!dist_less(best_d, dist)) {"),
    "quantize_8bit_float64_distance": ("return x.hi < y.hi || (x.hi == y.hi && x.lo < y.lo);",
                                       "return x.hi < y.hi;"),
    "quantize_8bit_absmax_without_abs": ("const float mag = fabsf(load_elem(x, dtype, i));",
                                         "const float mag = load_elem(x, dtype, i);"),
    "dequantize_8bit_skips_fp32_rounding": (
        "store_elem(out, out_dtype, i, entry * scale);",
        "if (out_dtype == ORACLE_BF16) ((uint16_t *)out)[i] = encode_format(round_to_format("
        "(double)entry * (double)scale, 8, -126, ldexp(2.0 - ldexp(1.0, -7), 127)), 7, 127, -126, 255);"
        " else store_elem(out, out_dtype, i, entry * scale);"),
    "embedding_rows_transposed": ("const int64_t e = idx[r] * D + k;", "const int64_t e = k * V + idx[r];"),
    "embedding_rows_in_reverse_order": ("store_elem(out, out_dtype, r * D + k,",
                                        "store_elem(out, out_dtype, (n_idx - 1 - r) * D + k,"),
}

PIN_CHECKS = [
    lambda: pins.test_worked_example_golden(),
    lambda: pins.test_nf4_table_matches_golden_literals_and_invariants(),
    lambda: pins.test_fp4_table_closed_form(),
    lambda: pins.test_special_blocks(),
    lambda: [pins.test_ties_go_to_smallest_index(q) for q in ("nf4", "fp4")],
    lambda: [pins.test_quantize_matches_exact_bruteforce(d, 130, 64, 5, q)
             for d in ("f32", "bf16") for q in ("nf4", "fp4")],
    lambda: [pins.test_division_knife_edges_match_exact_quotient(q) for q in ("nf4", "fp4")],
    lambda: [pins.test_dequant_double_rounding_edges(q, o) for q in ("nf4", "fp4") for o in ("bf16", "f16")],
    lambda: pins.test_f32_to_16bit_rne_against_torch_and_numpy(),
    lambda: pins.test_matmul_one_hot_gives_weight_column(),
    lambda: [pins.test_matmul_and_backward_exact_bruteforce(q) for q in ("nf4",)],
    lambda: [dq_pins.test_double_quant_matches_exact_rationals(g) for g in (4, 7, 256)],
    lambda: dq_pins.test_double_quant_closed_forms(),
    lambda: dq_pins.test_double_quant_special_values(),
    lambda: [q8_pins.test_matches_exact_rationals(k, "f32", 65, 64) for k in ("uniform", "log")],
    lambda: q8_pins.test_dyadic_linear_table_closed_form(),
    lambda: [q8_pins.test_every_midpoint_neighbourhood(k) for k in ("uniform", "log")],
    lambda: q8_pins.test_special_blocks(),
    lambda: q8_pins.test_symmetric_pair_decides_tiny_quotients_by_sign(),
    lambda: q8_pins.test_dequant_double_rounding(),
    lambda: [emb_pins.test_matches_exact_rationals(q, D, B) for q in ("nf4", "fp4") for D, B in ((12, 4), (13, 4))],
    lambda: emb_pins.test_index_checks(),
]


def _build_mutant(tmp, before, after):
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation anchor not unique: {before!r}"
    d = os.path.join(tmp, "m")
    os.makedirs(d)
    shutil.copy(os.path.join(os.path.dirname(SRC), "bnb4_oracle.h"), d)
    with open(os.path.join(d, "bnb4_oracle.c"), "w") as f:
        f.write(src.replace(before, after))
    so = os.path.join(d, "libmutant.so")
    subprocess.check_call(["cc", "-O1", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
                           "-shared", "-fPIC", "-o", so, os.path.join(d, "bnb4_oracle.c"), "-lm"])
    return so


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    before, after = MUTATIONS[name]
    with tempfile.TemporaryDirectory() as tmp:
        so = _build_mutant(tmp, before, after)
        real = oracle.lib()
        mutant = ctypes.CDLL(so)
        # same signatures as the real library
        for attr in ("oracle_code_table", "oracle_to_f32_array", "oracle_from_f32_array",
                     "oracle_quantize", "oracle_dequantize", "oracle_matmul",
                     "oracle_matmul_entries", "oracle_matmul_backward",
                     "oracle_matmul_backward_entries", "oracle_double_quant",
                     "oracle_dequant_absmax", "oracle_quantize_8bit", "oracle_dequantize_8bit",
                     "oracle_embedding_4bit"):
            f, g = getattr(real, attr), getattr(mutant, attr)
            g.restype, g.argtypes = f.restype, f.argtypes
        monkeypatch.setattr(oracle, "_lib", mutant)
        caught = 0
        for check in PIN_CHECKS:
            try:
                check()
            except (AssertionError, ValueError, pytest.fail.Exception):
                caught += 1
        assert caught > 0, f"no pin caught mutation {name}"
