"""CPU: the pins are strong enough to catch plausible mistakes in the oracle.

Each case plants one mistake in a temporary copy of the oracle's C source
(a dropped term, a wrong sign or index, a swapped operand), compiles it, and
requires that at least one pin rejects the broken copy.  The real oracle source
is never modified.
"""
import os

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "gqa_oracle.c")

MUTANTS = {
    "scale_dropped": ("s[i] = scale * dot;", "s[i] = dot;"),
    "exp_sign_flipped": ("double w = exp(s[i] - m);", "double w = exp(m - s[i]);"),
    "max_pass_dropped": ("if (s[i] > m)\n            m = s[i];", "m = 0.0;"),
    "head_map_modulo": ("int b = (int)(r / Hq), h = (int)(r % Hq);\n        int kvh = h / G;",
                        "int b = (int)(r / Hq), h = (int)(r % Hq);\n        int kvh = h % Hkv;"),
    "states_head_map_modulo": ("b, h / G, t0, t1", "b, h % Hkv, t0, t1"),
    "page_offset_shifted": ("offset = t % c->block_size;", "offset = (t + 1) % c->block_size;"),
    "block_index_shifted": ("t / c->block_size];", "(t / c->block_size) ^ 1];"),
    "key_replaced_by_value": ("dot += bf16_to_double(qrow[d]) * key_at(c, row + d);",
                              "dot += bf16_to_double(qrow[d]) * value_at(c, row + d);"),
    "e4m3_bias_off_by_one": ("ldexp(1.0 + (double)m / 8.0, e - 7)", "ldexp(1.0 + (double)m / 8.0, e - 8)"),
    "e4m3_subnormal_exponent": ("ldexp((double)m / 8.0, -6)", "ldexp((double)m / 8.0, -7)"),
    "e4m3_mantissa_width": ("1.0 + (double)m / 8.0, e - 7", "1.0 + (double)m / 16.0, e - 7"),
    "fp8_value_scale_dropped": ("e4m3_to_double(c->v8[i]) * c->v_scale", "e4m3_to_double(c->v8[i])"),
    "fp8_key_scale_dropped": ("e4m3_to_double(c->k8[i]) * c->k_scale", "e4m3_to_double(c->k8[i])"),
    "first_key_skipped": ("for (int64_t i = 0; i < n; ++i) {\n        double w",
                          "for (int64_t i = 1; i < n; ++i) {\n        double w"),
    "normaliser_unweighted": ("l += w;", "l += 1.0;"),
    "query_head_zero": ("rc = attention_state(&c, q + r * D, scale, b, kvh, 0, L, o, &m, &l);",
                        "rc = attention_state(&c, q + (r / Hq) * Hq * D, scale, b, kvh, 0, L, o, &m, &l);"),
    "multi_mask_off_by_one": ("0, L - Q + i + 1, o,", "0, L - Q + i, o,"),
    "multi_token_order": ("int b = (int)(bi / Q), i = (int)(bi % Q);",
                          "int i = (int)(bi / B), b = (int)(bi % B);"),
    "multi_mask_reversed": ("0, L - Q + i + 1, o,", "0, L - i, o,"),
    "merge_weight_sign": ("exp(mi - mstar)", "exp(mstar - mi)"),
    "merge_normaliser_unweighted": ("lstar += w * l[", "lstar += l["),
    "merge_lse_dropped_max": ("mstar + log(lstar)", "log(lstar)"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    lib = oracle.build(force=True, src=str(path), lib=str(tmp_path / "libmutant.so"))
    bad = oracle.Oracle(lib)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(bad)
        except Exception:   # an AssertionError, or an error the mutant raises
            caught.append(pin.__name__)
    assert caught, f"no pin rejects mutant {name}"
