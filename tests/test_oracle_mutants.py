"""Planted mistakes in copies of the oracle source must be caught by a pin.

Each mutant is a one-line textual change of ``oracle/ternary_oracle.c`` — a
dropped term, a wrong sign or index, a wrong rounding mode, a missing clip or
floor, a wrong scale — compiled with the oracle's own flags into a temporary
library.  Every pin in ``oracle_pins.py`` is run against it, and at least one
must fail.  The real oracle is never modified.
"""
import os

import pytest

from oracle import oracle as orc
from tests.oracle_pins import ALL_PINS

MUTANTS = {
    "half_away_codes": ("double r = rint((double)W[i] * s);",
                        "double r = round((double)W[i] * s);"),
    "half_away_q": ("float r = rintf(v);", "float r = roundf(v);"),
    "no_clip": ("if (r > 1.0)\n            r = 1.0;",
                "if (r > 2.0)\n            r = 2.0;"),
    "s_not_reciprocal": ("double s = 1.0 / mean;", "double s = mean;"),
    "scale_128": ("float scale = 127.0f / a;\n        for (int64_t k = 0; k < K; ++k) {\n            float v",
                  "float scale = 128.0f / a;\n        for (int64_t k = 0; k < K; ++k) {\n            float v"),
    "drop_last_term": ("for (int64_t k = 0; k < K; ++k)\n                sum +=",
                       "for (int64_t k = 0; k < K - 1; ++k)\n                sum +="),
    "sign_flip": ("sum += (int64_t)codes", "sum -= (int64_t)codes"),
    "token_index": ("(int64_t)q[m * K + k]", "(int64_t)q[(M - 1 - m) * K + k]"),
    "weight_row_index": ("(int64_t)codes[n * K + k]",
                         "(int64_t)codes[(N - 1 - n) * K + k]"),
    "rescale_no_127": ("double a = (double)amax[m] / 127.0;",
                       "double a = (double)amax[m];"),
    "rescale_div_mean": ("(double)acc[m * N + n] * a * mean;",
                         "(double)acc[m * N + n] * a / mean;"),
    "mean_over_N": ("double mean = total / (double)(N * K);",
                    "double mean = total / (double)(N);"),
    "no_abs": ("row += fabs((double)W[n * K + k]);",
               "row += ((double)W[n * K + k]);"),
    "no_floor": ("if (mean < ORC_MEAN_FLOOR)\n        mean = ORC_MEAN_FLOOR;", ""),
    "amax_signed": ("float v = fabsf(row[k]);", "float v = row[k];"),
    "fp32_row_sum": ("double row = 0.0;", "float row = 0.0f;"),
    "gqa_head_mod": ("(h / group) * head_dim + c]", "(h % n_kv) * head_dim + c]"),
    "add_subtracts": ("out[i] = x[i] + y[i];", "out[i] = x[i] - y[i];"),
    "silu_sign": ("z / (1.0 + exp(-z))", "z / (1.0 + exp(z))"),
    "silu_drops_u": ("exp(-z)) * (double)u[i];", "exp(-z));"),
    "i8_no_relu": ("if (relu && v < 0.0)", "if (0 && v < 0.0)"),
    "i8_bias_subtracted": ("v += (double)bias[n];", "v -= (double)bias[n];"),
    "i8_bias_first_only": ("v += (double)bias[n];", "v += (double)bias[0];"),
    "i8_weight_scale_no_127": ("const double w = (double)amax_w / 127.0;",
                               "const double w = (double)amax_w;"),
    "i8_token_scale_no_127": ("const double a = (double)amax_x[m] / 127.0;",
                              "const double a = (double)amax_x[m] / 128.0;"),
    "given_scale_128": ("const float scale = 127.0f / a;", "const float scale = 128.0f / a;"),
    "i8_relu_clamps_above": ("if (relu && v < 0.0)\n                v = 0.0;",
                             "if (relu && v > 0.0)\n                v = 0.0;"),
}
# Not listed: removing the amax == 0 special cases (of orc_quantize_act and
# orc_quantize_act_given).  On x86-64 the resulting NaN converts to 0 anyway,
# so those mutants are equivalent and uncatchable; the special cases stay
# because the conversion of NaN is undefined in C.


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = orc.source_text()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    lib_path = orc.compile_variant(src.replace(old, new),
                                   os.path.join(tmp_path, f"mut_{name}.so"))
    prev = orc.use_library(lib_path)
    caught = []
    try:
        for pin_name, pin in ALL_PINS.items():
            try:
                pin()
            except (AssertionError, ValueError, OverflowError):
                caught.append(pin_name)
    finally:
        orc.use_library(prev)
    assert caught, f"mutant {name} passed every pin"
