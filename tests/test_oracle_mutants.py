"""Planted mistakes in a copy of the oracle must each fail at least one pin.

The mistakes are planted in a temporary copy of the oracle's C source (never
in the CUDA path), compiled with the same flags, and run against every pin.
A mutant that passes every pin would mean the pins cannot see that mistake.
"""
import os

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "int8lt_oracle.c")

# (name, original text, planted mistake)
MUTANTS = [
    ("round_floor", "float r = nearbyintf(p);", "float r = floorf(p);"),
    ("round_half_away", "float r = nearbyintf(p);", "float r = roundf(p);"),
    ("round_trunc", "float r = nearbyintf(p);", "float r = truncf(p);"),
    ("outlier_strict_gt", "if (ax >= threshold) hit = 1;", "if (ax > threshold) hit = 1;"),
    ("row_scale_includes_outliers", "if (mask && mask[h]) continue;", "if (0) continue;"),
    ("outlier_codes_not_zeroed", "if (mask && mask[h]) { q[h] = 0; continue; }", "if (0) { q[h] = 0; continue; }"),
    ("dequant_missing_127", "/ 16129.0", "/ 127.0"),
    ("dequant_missing_sca", "(double)acc * (double)sca * (double)SCB[j]", "(double)acc * (double)SCB[j]"),
    ("drop_outlier_product", "y += oracle_half_to_double(xrow[h]) *", "y += 0.0 *"),
    ("outlier_product_sign", "y += oracle_half_to_double(xrow[h]) *", "y -= oracle_half_to_double(xrow[h]) *"),
    ("drop_bias", "if (bias) y += oracle_half_to_double(bias[j]);", "if (bias) y += 0.0;"),
    ("outlier_weight_wrong_column", "return oracle_half_to_double(W_outlier[j * K + h]);",
     "return oracle_half_to_double(W_outlier[j * K + (K - 1 - h)]);"),
    ("recovery_div_128", "float u = t / 127.0f;", "float u = t / 128.0f;"),
    ("gemm_off_by_one", "for (int64_t k = 0; k < K; ++k) acc += (int64_t)a[k] * (int64_t)b[k];",
     "for (int64_t k = 1; k < K; ++k) acc += (int64_t)a[k] * (int64_t)b[k];"),
    ("forward_transposed_cb", "const int8_t *b = CB + j * K;", "const int8_t *b = CB + (N - 1 - j) * K;"),
    ("scale_127_wrong", "float s = 127.0f / absmax;", "float s = 128.0f / absmax;"),
    ("half_subnormal_exp", "v = ldexp((double)man, -24);", "v = ldexp((double)man, -25);"),
    ("half_encode_ties_away", "double r = nearbyint(ldexp(a, 10 - E));", "double r = round(ldexp(a, 10 - E));"),
    ("zp_drop_k_term", "+ K * (int64_t)za * ZPB[j];", ";"),
    ("zp_sign", "int64_t c = (int64_t)nearbyintf(h2f(x[h]) * nd) - z;", "int64_t c = (int64_t)nearbyintf(h2f(x[h]) * nd) + z;"),
    ("zp_ties_away", "int64_t c = (int64_t)nearbyintf(h2f(x[h]) * nd) - z;", "int64_t c = (int64_t)roundf(h2f(x[h]) * nd) - z;"),
    ("zp_range_255", "float nd = range > 0.0f ? 254.0f / range : 1.0f;", "float nd = range > 0.0f ? 255.0f / range : 1.0f;"),
    ("zp_no_shift", "int32_t z = (int32_t)zmin + 127;", "int32_t z = (int32_t)zmin;"),
    ("zp_correction_swapped", "(int64_t)ZPB[j] * sa + (int64_t)za * SUMB[j]", "(int64_t)za * sa + (int64_t)ZPB[j] * SUMB[j]"),
    ("weight_scale_wrong_row", "SCB[j] = quantize_vector(W + j * K, NULL, K, CB + j * K);",
     "SCB[j] = quantize_vector(W + j * K, NULL, K - 1, CB + j * K);"),
    ("forward_rows_ignores_subset", "int64_t i = rows[r];", "int64_t i = r;"),
    ("zp_forward_rows_ignores_subset", "zp_quantize_vector(X + rows[r] * K, K, ca, &za, &sa);",
     "zp_quantize_vector(X + r * K, K, ca, &za, &sa);"),
    ("forward_rows_outliers_from_subset",
     "int64_t n_out = oracle_outlier_columns(X, M, K, threshold, idx);",
     "int64_t n_out = oracle_outlier_columns(X + rows[0] * K, 1, K, threshold, idx);"),
]


@pytest.mark.parametrize("name,orig,bad", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, orig, bad):
    src = open(SRC).read()
    assert src.count(orig) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(orig, bad)
    c = tmp_path / f"{name}.c"
    c.write_text(mutated)
    so = oracle.build(str(c), str(tmp_path / f"lib{name}.so"), force=True)
    lib = oracle.load(so)
    failed = []
    for pin in oracle_pins.PINS:
        try:
            pin(lib)
        except (AssertionError, OverflowError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
