"""The CPU oracle against its pins (no GPU)."""
import pytest

from oracle import formats, quant, svd, svdquant
from tests import oracle_pins as P


def test_format_tables():
    P.pin_format_tables(formats)


def test_encoders_bruteforce():
    P.pin_encoders_bruteforce(formats)


def test_fp16_rounding_matches_numpy():
    P.pin_fp16_rounding(formats)


def test_bf16_rounding_exact():
    P.pin_bf16_rounding(formats)


def test_int4_golden_w4a8_formula():
    P.pin_int4_golden(quant)


def test_int4_bruteforce():
    P.pin_int4_bruteforce(quant)


def test_nvfp4_bounds():
    P.pin_nvfp4_bounds(quant, formats)


def test_svd_known_answers():
    P.pin_svd_known_answers(svd)


def test_svd_vs_lapack():
    P.pin_svd_vs_lapack(svd)


def test_eckart_young():
    P.pin_eckart_young(svd, svdquant)


def test_smoothing():
    P.pin_smoothing(svdquant)


def test_rank0_is_plain_rtn():
    P.pin_rank0_plain_rtn(svdquant)


def test_bruteforce_int4_exact():
    P.pin_bruteforce_int4(svdquant)


def test_bruteforce_nvfp4_exact():
    P.pin_bruteforce_nvfp4(svdquant)


def test_special_cases():
    P.pin_special_cases(svdquant)


def test_on_grid_lossless():
    P.pin_on_grid_lossless(svdquant)


def test_low_rank_branch_lowers_error():
    P.pin_low_rank_helps(svdquant)


def test_act_tensor_scale_golden():
    P.pin_act_tensor_scale_golden(svdquant)


def test_act_codes_from_smoothed_x_golden():
    P.pin_act_codes_golden(svdquant)


def test_act_tensor_scale_in_prepare():
    P.pin_act_scale_in_prepare(svdquant)


def test_lapack_factors_match_jacobi():
    P.pin_lapack_factors_match_jacobi(svdquant)


def test_next_layer_input_bruteforce():
    P.pin_next_layer_input_bruteforce(svdquant)
