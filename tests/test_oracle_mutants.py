"""Plant plausible mistakes in copies of the oracle and check that the pins catch every one.

Each mutant is the oracle's C source with one textual change, compiled into a
temporary directory on the CPU.  A mutant that passes every pin would mean
the pins cannot tell that mistake from the right answer.
"""

import pytest

import oracle
from tests import oracle_pins

MUTANTS = {
    "rope_first_half_sign": ("y[i] = a * c - b * s;", "y[i] = a * c + b * s;"),
    "rope_second_half_sign": ("y[i + half] = b * c + a * s;", "y[i + half] = b * c - a * s;"),
    "rope_interleaved_pairs": ("double a = x[i], b = x[i + half];\n    y[i] = a * c - b * s;\n    y[i + half] = b * c + a * s;",
                               "double a = x[2 * i], b = x[2 * i + 1];\n    y[2 * i] = a * c - b * s;\n    y[2 * i + 1] = b * c + a * s;"),
    "rope_freq_exponent": ("pow(base, -2.0 * (double)i / (double)D)", "pow(base, -1.0 * (double)i / (double)D)"),
    "query_position_L_minus_1": ("oracle_rope(xk, D, (double)L, rope_base", "oracle_rope(xk, D, (double)(L - 1), rope_base"),
    "key_position_plus_1": ("oracle_rope(xk, D, (double)t, rope_base, khat);", "oracle_rope(xk, D, (double)(t + 1), rope_base, khat);"),
    "gqa_interleaved_heads": ("const float* qr = q + ((size_t)b * Hq + (size_t)h * G + g) * D;",
                              "const float* qr = q + ((size_t)b * Hq + (size_t)g * Hkv + h) * D;"),
    "scale_dropped": ("s[(size_t)g * L + t] = sc * acc;", "s[(size_t)g * L + t] = acc;"),
    "softmax_unnormalised": ("double w = sg[t] / z;", "double w = sg[t];"),
    "f16_exponent_bias": ("mag = ldexp((double)(1024 + frac), expo - 25);", "mag = ldexp((double)(1024 + frac), expo - 24);"),
    "f16_subnormal_scale": ("mag = ldexp((double)frac, -24);", "mag = ldexp((double)frac, -25);"),
    "bf16_wrong_shift": ("uint32_t u = ((uint32_t)b) << 16;", "uint32_t u = ((uint32_t)b) << 15;"),
    "v_read_from_k": ("o[d] += w * decode16(vb[(size_t)t * D + d], kv_dtype);",
                      "o[d] += w * decode16(kb[(size_t)t * D + d], kv_dtype);"),
    "projection_transposed": ("decode16(w[(size_t)r * H + h], kv_dtype) * (double)x[(size_t)b * H + h]",
                              "decode16(w[(size_t)h * R + r], kv_dtype) * (double)x[(size_t)b * H + h]"),
    "last_token_dropped": ("for (int64_t t = 0; t < L; ++t) {\n        double w", "for (int64_t t = 0; t + 1 < L; ++t) {\n        double w"),
}

# cheapest pins first: each mutant stops at the first pin that catches it
ORDER = sorted(oracle_pins.ALL_PINS, key=lambda f: ("decode" in f.__name__, f.__name__ == "pin_rope_vs_hf"))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = oracle.SRC.read_text()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutant_src = tmp_path / "mutant.c"
    mutant_src.write_text(src.replace(old, new))
    lib = oracle.load(oracle.build(force=True, src=mutant_src, out=tmp_path / "libmutant.so"))
    caught_by = None
    for pin in ORDER:
        try:
            pin(lib)
        except AssertionError:
            caught_by = pin.__name__
            break
    del lib
    assert caught_by is not None, f"mutant {name} passed every pin"
