"""Planted mistakes: each mutant of the oracle (one plausible error compiled
in with -DWQO_MUTANT=k) must fail at least one pin, and the real oracle must
pass the same pins.  This shows the pins constrain every step: statistics,
scale, zero point, rounding, 4- and 8-bit packing, dequantization (zero point and
bf16 rounding), the linear layer (operand, sum range, error scale) and
the clipping search (error formula, candidate ranges and selection), the AWQ
scales and scaled activations, GPTQ (pivot division, tail update, processing
order, dampening), the symmetric scale and nibble sign, and the code of NaN."""
import pytest

import oracle
from tests import test_oracle_awq_pins as awq_pins
from tests import test_oracle_clip_pins as clip_pins
from tests import test_oracle_gptq_pins as gptq_pins
from tests import test_oracle_pins as pins

PINS = [
    pins.test_zero_exactly_representable,
    pins.test_outlier20_symmetric,
    lambda: pins.test_round_trip_fixed_point(True),
    pins.test_degenerate_and_nonfinite_groups,
    lambda: pins.test_rounding_error_bound(False),
    pins.test_outlier20_asymmetric_and_clipping,
    lambda: pins.test_round_trip_fixed_point(False),
    lambda: pins.test_brute_force_argmin(-1.0, 1.5, False),
    lambda: pins.test_brute_force_argmin(0.25, 7.0, False),
    pins.test_pack_layout_low_nibble_first,
    pins.test_pack8_layout_low_byte_first,
    pins.test_dequant_exhaustive_against_library_rounding,
    pins.test_linear_special_cases_and_matmul,
    clip_pins.test_error_formula_is_the_exact_sum_of_squares,
    clip_pins.test_choice_is_the_exact_argmin,
    clip_pins.test_never_worse_than_rtn,
    awq_pins.test_scales_follow_the_page_formula,
    awq_pins.test_losses_and_choice_recomputed_independently,
    gptq_pins.test_factor_is_the_upper_cholesky_of_the_damped_inverse_hessian,
    lambda: gptq_pins.test_codes_match_an_independent_unblocked_sweep(gptq_pins.CASES[0]),
    gptq_pins.test_obq_two_column_step,
    gptq_pins.test_damping_is_one_percent_of_the_mean_diagonal,
]

MUTANTS = {
    1: "zero point sign",
    2: "round half away from zero",
    3: "scale divided by level count",
    4: "range not widened to zero",
    5: "transposed weight in linear",
    6: "zero point dropped in dequant",
    7: "high nibble first",
    8: "8-bit packing high byte first",
    9: "clip search sums absolute errors",
    10: "clip search keeps the largest error",
    11: "AWQ scales inverted",
    12: "GPTQ error not divided by the pivot",
    13: "GPTQ tail update reads the factor transposed",
    14: "GPTQ act-order ascending",
    15: "symmetric scale over eight",
    16: "symmetric nibbles not sign extended",
    17: "NaN takes the lowest code",
    18: "GPTQ dampening missing",
    19: "AWQ scales not normalised by the geometric mean",
    20: "clip search shrinks only the upper end",
    21: "AWQ activations multiplied by s",
    22: "linear drops the last input channel",
    23: "linear error scale sums signed terms",
    24: "dequant truncates to bf16",
}


def _failures():
    n = 0
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            n += 1
    return n


@pytest.mark.parametrize("mutant", sorted(MUTANTS), ids=lambda m: MUTANTS[m].replace(" ", "-"))
def test_mutant_is_caught(mutant, tmp_path):
    path = oracle.build_mutant(mutant, str(tmp_path))
    with oracle.use_library(path):
        assert _failures() >= 1, MUTANTS[mutant]


def test_real_oracle_passes_the_same_pins():
    assert _failures() == 0
