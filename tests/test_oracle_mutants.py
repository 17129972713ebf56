"""The oracle's pins are strong enough: each plausible mistake, planted in a
copy of the C oracle (never in the real one), makes at least one pin fail."""
import os

import pytest

import oracle
from test_oracle_pins import PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "skipsoftmax_oracle.c")

MUTANTS = {
    "non_strict_compare": ("const int skip = margin < 0.0;", "const int skip = margin <= 0.0;"),
    "any_row_instead_of_every_row": (
        "if (x > margin) margin = x;",
        "if (margin == -INFINITY || x < margin) margin = x;"),
    "tile0_skippable": ("if (m == -INFINITY) return INFINITY;", "if (m == -INFINITY) return -INFINITY;"),
    "tau_in_log2_units": ("return mt - m + tau;", "return mt - m + tau * 1.4426950408889634;"),
    "missing_scale": ("d) * inv_sqrt_d;\n                s[", "d);\n                s["),
    "exp2_instead_of_exp": ("const double p = exp(x - m_new);", "const double p = exp2(x - m_new);"),
    "sum_not_rescaled": ("            l[r] *= alpha;\n            double *ar", "            double *ar"),
    "acc_not_rescaled": ("for (int t = 0; t < d; ++t) ar[t] *= alpha;", ""),
    "kv_head_modulo": ("const int kvh = h / g;", "const int kvh = h % a->Hkv;"),
    "causal_off_by_one": ("if (a->causal && c > qi) x = -INFINITY;", "if (a->causal && c >= qi && qi > 0) x = -INFINITY;"),
    "transposed_value_rows": ("ar[t] += p * widen_bf16(vc[t]);", "ar[t] += p * widen_bf16(v[(size_t)t * d + (c % d)]);"),
    "decode_max_not_reset_per_split": (
        "for (int r = 0; r < g; ++r) { m[r] = seeded ? seed[r] : -INFINITY; l[r] = 0.0; }\n            for (size_t t",
        "for (int r = 0; r < g; ++r) { if (sp == 0) m[r] = seeded ? seed[r] : -INFINITY; l[r] = 0.0; }\n            for (size_t t"),
    "decode_merge_unweighted_sum": ("den += w * sl[(size_t)sp * g + r];", "den += sl[(size_t)sp * g + r];"),
    "per_head_uses_group_margin": (
        "if (per_head && row_margin(mt[r], m[r], tau) < 0.0) {",
        "if (per_head && margin_j < 0.0) {"),
    "e4m3_ties_to_odd": ("((lo + 1) & 1) == 0)", "((lo + 1) & 1) == 1)"),
    "e4m3_ties_away_from_zero": ("(dh == dl && ((lo + 1) & 1) == 0)", "(dh == dl)"),
    "e4m3_subnormal_exponent": ("v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    "e4m3_scale_not_smallest": ("while (amax > ldexp(448.0, k))", "while (amax >= ldexp(448.0, k))"),
    "e4m3_sign_dropped": ("? 0x80 : 0));", "? 0x00 : 0));"),
    "i8_ties_upward": ("(fmod(f, 2.0) == 0.0) ? f : f + 1.0", "f + 1.0"),
    "i8_scale_not_smallest": ("while (amax > ldexp(127.0, k))", "while (amax >= ldexp(127.0, k))"),
    "i8_range_128": ("while (amax > ldexp(127.0, k))", "while (amax > ldexp(128.0, k))"),
    "sink_seed_from_second_tile": (
        "for (int c = 0; c < Bt && c < L; ++c)", "for (int c = Bt; c < 2 * Bt && c < L; ++c)"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) >= 1, f"mutation site for {name} not found"
    src = tmp_path / f"mut_{name}.c"
    src.write_text(text.replace(old, new, 1))
    lib = oracle.build(force=True, src=str(src), out=str(tmp_path / f"lib_{name}.so"))
    caught = []
    for fn in PINS:
        try:
            fn(lib)
        except (AssertionError, ValueError):
            caught.append(fn.__name__)
            break
    assert caught, f"no pin catches the planted mistake {name}"
