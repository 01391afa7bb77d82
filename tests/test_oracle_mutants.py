"""Mutation check of the oracle's pins.  Each mutant below is one plausible
mistake (a wrong tie rule, index, sign, operand, constant, comparison or
rounding) planted in a copy of oracle/mxq_oracle.c on the CPU; the copy is
built with the oracle's own flags and swapped in, and the pins of
tests/test_oracle_*.py run against it until one fails.  Every mutant must be
caught: a mutant that survives marks a part of the oracle that no pin
fixes."""
import importlib
import subprocess

import pytest

import oracle
from oracle import capi

MUTANTS = [
    ("ties_go_to_m4", "use4 = (G4 < G6);", "use4 = (G4 <= G6);"),
    ("s2_without_the_6", "float s2 = amax_g / (float)global_div;",
     "float s2 = amax_g / (float)(global_div / 6.0);"),
    ("plan_divides_twice", "float t = amax_b / den;", "float t = (amax_b / M) / s2; (void)den;"),
    ("ties_to_the_larger_code", "(dist == best_dist && (c & 1u) == 0u)", "(dist == best_dist && c > best)"),
    ("nibbles_swapped", "codes[gb * 8 + j] = (uint8_t)((c[2 * j] & 0xF) | ((c[2 * j + 1] & 0xF) << 4));",
     "codes[gb * 8 + j] = (uint8_t)((c[2 * j + 1] & 0xF) | ((c[2 * j] & 0xF) << 4));"),
    ("mx_exponent_not_strict", "while (e < 127 && amax > ldexp(qmax, e))",
     "while (e < 127 && amax >= ldexp(qmax, e))"),
    ("e4m3_subnormal_exponent", "mag = ldexp((double)m / 8.0, -6);", "mag = ldexp((double)m / 8.0, -7);"),
    ("e2m1_subnormal_value", "mag = 0.5 * (double)m;", "mag = 0.25 * (double)m;"),
    ("values_use_the_ideal_scale", "\n        d = (float)D * s2;", "\n        d = amax_b / M;"),
    ("plan4_uses_divisor_6", "r = nvfp4_plan(xb, amax_b, s2, 4.0f, &sc4, c4, &G4);",
     "r = nvfp4_plan(xb, amax_b, s2, 6.0f, &sc4, c4, &G4);"),
    ("decision_sign_of_A", "double P = exact_add(exact_mul(dS, B, &ok), -2.0 * A, &ok);",
     "double P = exact_add(exact_mul(dS, B, &ok), 2.0 * A, &ok);"),
    ("group_amax_without_abs",
     "float v = fabsf(bf16_to_float(xg[i]));\n            if (!isfinite(v))\n                return -3;\n"
     "            if (v > amax_g)\n                amax_g = v;\n        }\n        float s2",
     "float v = bf16_to_float(xg[i]);\n            if (!isfinite(v))\n                return -3;\n"
     "            if (v > amax_g)\n                amax_g = v;\n        }\n        float s2"),
    ("mx_block_amax_without_abs", "if (fabs(v[i]) > amax)\n                amax = fabs(v[i]);",
     "if (v[i] > amax)\n                amax = v[i];"),
    ("verifier_s2_per_tensor", "(double)s2[t / tensors_per_scale];", "(double)s2[t];"),
    ("verifier_mxfp4_scale_index", "deq = q * oracle_ue8m0_value(scales[gi / 32]);",
     "deq = q * oracle_ue8m0_value(scales[gi / 16]);"),
    ("verifier_ref_from_deq", "ref += xv * xv;", "ref += deq * deq;"),
    ("requant_scale_column", "bscale[(r / brows) * nbc + c / bcols]", "bscale[(r / brows) * nbc + c / brows]"),
    ("weighted_ties_to_the_larger_code", "if (w < best_w) {", "if (w <= best_w) {"),
    ("weighted_candidates_stop_short", "for (unsigned sc = lo + 1; sc <= hi; ++sc) {",
     "for (unsigned sc = lo + 1; sc < hi; ++sc) {"),
    ("s2_by_reciprocal", "float s2 = amax_g / (float)global_div;",
     "float s2 = amax_g * (float)(1.0 / global_div);"),
    ("quotient_by_reciprocal", "float y = x[i] / d;", "float y = x[i] * (1.0f / d);"),
    ("requant_product_not_rounded", ("float w[32];", "w[i] = (float)(oracle_e4m3_value(q) * (double)sc);"),
     ("double w[32];", "w[i] = oracle_e4m3_value(q) * (double)sc;")),
]


def _pins():
    c, n, m, r, w = (importlib.import_module("test_oracle_" + k)
                     for k in ("codecs", "nvfp4", "mx_verifier", "requant", "weighted"))
    o = oracle
    return [
        lambda: c.test_e2m1_decode_matches_golden_grid(o),
        lambda: c.test_e2m1_ties_golden(o),
        lambda: c.test_e2m1_encode_at_every_midpoint_and_neighbours(o),
        lambda: c.test_e4m3_decode_golden_points(o),
        lambda: c.test_e4m3_round_trip_and_saturation(o),
        lambda: c.test_mx_exponent_golden(o),
        lambda: n.test_worked_example_golden(o),
        lambda: n.test_global_scale_closed_form_and_amax_block_scale(o),
        lambda: n.test_gate_up_share_one_weight_scale_2(o),
        lambda: n.test_block_scale_divides_the_amax_once(o),
        lambda: n.test_values_take_the_ieee_quotient_at_e2m1_ties(o),
        lambda: n.test_blocks_match_exact_rational_micro_oracle(o, 1.0),
        lambda: n.test_ties_keep_the_amax6_plan(o),
        lambda: n.test_rtn_mode_equals_plan6_of_four_six(o),
        lambda: n.test_metamorphic_scaling_sign_and_permutation(o),
        lambda: n.test_exact_decision_values_match_rational_sse(o),
        lambda: m.test_mx_scale_satisfies_exponent_rule_per_block(o),
        lambda: m.test_mx_values_are_nearest_codes(o),
        lambda: m.test_mxfp8_relerr_matches_published_sanity_band(o),
        lambda: m.test_relerr_zero_for_exactly_representable_input(o),
        lambda: m.test_nvfp4_verifier_reads_shared_scale_per_fused_slab(o),
        lambda: m.test_relerr_matches_independent_numpy_dequant(o),
        lambda: r.test_hand_worked_block(),
        lambda: r.test_dequantized_value_is_rounded_to_fp32_once(),
        lambda: r.test_bf16_exact_case_reduces_to_the_bf16_quantizer("mxfp4"),
        lambda: w.test_matches_the_exact_argmin_away_from_near_ties(),
        lambda: w.test_one_hot_weight_reproduces_that_element_best(0),
    ]


def test_unmutated_oracle_passes_every_pin_used_here():
    for pin in _pins():
        pin()


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, monkeypatch, name, old, new):
    with open(capi._SRC) as f:
        src = f.read()
    olds, news = (old, new) if isinstance(old, tuple) else ((old,), (new,))
    for o, n in zip(olds, news):
        assert src.count(o) == 1, "the mutated text must occur exactly once"
        src = src.replace(o, n)
    c_path, so_path = tmp_path / (name + ".c"), tmp_path / (name + ".so")
    c_path.write_text(src)
    subprocess.check_call(["gcc", *capi.CFLAGS, "-o", str(so_path), str(c_path), "-lm"])
    monkeypatch.setattr(capi, "_lib", capi.load_library(str(so_path)))
    for pin in _pins():
        try:
            pin()
        except (AssertionError, RuntimeError, ValueError):
            return                                  # caught
    pytest.fail("mutant %s passed every pin" % name)


# ---- the tiled scale layout (oracle/layout.py) ----------------------------
def _rows_one_after_another(r, c, cols):
    n = -(-cols // 4)
    return ((r // 128) * n + c // 4) * 512 + 4 * (r % 128) + c % 4


def _column_and_slab_swapped(r, c, cols):
    n, rr = -(-cols // 4), r % 128
    return ((r // 128) * n + c // 4) * 512 + 16 * (rr % 32) + (rr // 32) + 4 * (c % 4)


def _line_and_slab_strides_swapped(r, c, cols):
    n, rr = -(-cols // 4), r % 128
    return ((r // 128) * n + c // 4) * 512 + 4 * (rr % 32) + 16 * (rr // 32) + c % 4


def _column_tiles_rounded_down(r, c, cols):
    n, rr = max(cols // 4, 1), r % 128
    return ((r // 128) * n + c // 4) * 512 + 16 * (rr % 32) + 4 * (rr // 32) + c % 4


@pytest.mark.parametrize("mutant", [_rows_one_after_another, _column_and_slab_swapped,
                                    _line_and_slab_strides_swapped, _column_tiles_rounded_down],
                         ids=lambda f: f.__name__.strip("_"))
def test_layout_mutant_is_caught(monkeypatch, mutant):
    from oracle import layout
    lay = importlib.import_module("test_oracle_layout")
    monkeypatch.setattr(layout, "tile_offset", mutant)
    pins = [lay.test_hand_worked_offsets,
            lambda: lay.test_bijection_onto_padded_matrix(130, 5),
            lambda: lay.test_tiles_are_contiguous_submatrices_and_padding_is_zero(128, 4),
            lay.test_round_trip_and_vectorised_path]
    for pin in pins:
        try:
            pin()
        except (AssertionError, IndexError):
            return
    pytest.fail("layout mutant %s passed every pin" % mutant.__name__)
