"""Plant plausible mistakes in a copy of the C oracle (CPU only) and check that
at least one pin fails for each: the pins are strong enough to catch a dropped
term, a wrong sign, index or layout, a transposed operand or a wrong rounding."""

import os

import pytest

from oracle import build as obuild
from oracle.ref import COracle
from pins import ALL_PINS

SRC = open(obuild.SRC).read()

MUTANTS = {
    "ternary_round_half_even": ("return (int)roundf(t);", "return (int)rintf(t);"),
    "act_round_half_even": ("float r = roundf(v);", "float r = rintf(v);"),
    "layout_transposed": ("return 8 * i + 2 * j;", "return 2 * i + 8 * j;"),
    "minus_one_sign": ("case 2: return -1;", "case 2: return 1;"),
    "code_table_swapped": ("return q == 0 ? 0u : (q > 0 ? 1u : 2u);",
                           "return q == 0 ? 0u : (q > 0 ? 2u : 1u);"),
    "gamma_drops_abs": ("row += fabs((double)W[n * K + k]);", "row += (double)W[n * K + k];"),
    "gamma_wrong_count": ("return (float)(total / (double)(N * K));",
                          "return (float)(total / (double)(K));"),
    "gamma_drops_last_row": ("for (int64_t n = 0; n < N; ++n) {\n        double row",
                             "for (int64_t n = 0; n < N - 1; ++n) {\n        double row"),
    "act_scale_128": ("float sm = 127.0f / amax;", "float sm = 128.0f / amax;"),
    "act_clamp_126": ("if (r > 127.0f) r = 127.0f;", "if (r > 126.0f) r = 126.0f;"),
    "act_zero_row_scale": ("s[m] = 1.0f;", "s[m] = 0.0f;"),
    "dot_reversed_k": ("sum += (int64_t)xq[m * K + k] * v;",
                       "sum += (int64_t)xq[m * K + (K - 1 - k)] * v;"),
    "epilogue_transposed": ("float r = gamma / s[m];", "float r = s[m] / gamma;"),
    "relu2_no_square": ("v = v * v;", "v = v;"),
    "relu_dropped": ("v = v > 0.0f ? v : 0.0f;", "v = v;"),
    "bf16_round_half_up": ("u += 0x7fffu + ((u >> 16) & 1u);", "u += 0x8000u;"),
    "gamma_zero_guard_dropped": ("if (gamma == 0.0f)\n        return 0;\n    float t", "float t"),
    "ternary_threshold_shift": ("float t = w / gamma;", "float t = w / gamma * 0.9f;"),
    "rms_norm_drops_eps": ("sqrt(ss / (double)K + 1e-6)", "sqrt(ss / (double)K)"),
    "rms_norm_sum_not_mean": ("sqrt(ss / (double)K + 1e-6)", "sqrt(ss + 1e-6)"),
    "rms_norm_no_sqrt": ("(float)(1.0 / sqrt(ss / (double)K + 1e-6))",
                         "(float)(1.0 / (ss / (double)K + 1e-6))"),
    "rms_norm_k_minus_one": ("sqrt(ss / (double)K + 1e-6)", "sqrt(ss / (double)(K - 1) + 1e-6)"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    assert SRC.count(old) == 1, f"mutation site not unique: {old!r}"
    lib = obuild.build_variant(SRC.replace(old, new), os.path.join(tmp_path, f"m_{name}.so"))
    R = COracle(lib)
    failed = []
    for pin in ALL_PINS:
        try:
            pin(R)
        except AssertionError:
            failed.append(pin.__name__)
        except Exception:  # an oracle error status also counts as caught
            failed.append(pin.__name__ + "(error)")
    assert failed, f"no pin catches mutant {name}"
