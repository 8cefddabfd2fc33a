"""The CPU oracle against what the pages and the mathematics fix (no GPU)."""

import oracle
import oracle_pins as P
from oracle import attention, codebook, quantize, rng, rotation


def test_splitmix64_published_outputs():
    P.pin_splitmix64(rng)


def test_sign_balance():
    P.pin_sign_balance(rng)


def test_first_rotation_signs():
    P.pin_first_signs(rng)


def test_first_qjl_pair():
    P.pin_first_qjl_pair(rng)


def test_qjl_matrix_is_gaussian():
    P.pin_qjl_gaussian(rng)


def test_hadamard_matches_scipy():
    P.pin_hadamard(rotation)


def test_rotation_orthogonal_and_invertible():
    P.pin_rotation_orthogonal(rotation, rng)


def test_rotation_basis_closed_form():
    P.pin_rotation_basis(rotation, rng)


def test_density_moments():
    P.pin_density_moments(codebook)


def test_codebook_uniform_density_case():
    P.pin_uniform_case(codebook)


def test_codebook_one_bit_closed_form():
    P.pin_one_bit_closed_form(codebook)


def test_codebook_centroid_condition():
    P.pin_centroid_condition(codebook)


def test_codebook_gaussian_limit_matches_max_1960():
    P.pin_gaussian_limit(codebook)


def test_distortion_identity_and_page_bound():
    P.pin_distortion(codebook)


def test_pack_matches_bigint_bitstream():
    P.pin_pack_bigint(quantize)


def test_codes_are_nearest_centroid():
    P.pin_codes_nearest(quantize, codebook, rng)


def test_dequantisation_is_nearest_reconstruction():
    P.pin_dequant_nearest(quantize, codebook, rng)


def test_int8_worked_cases():
    P.pin_int8_cases(quantize)


def test_qjl_residual_removes_inner_product_bias():
    P.pin_qjl_unbiased(quantize, codebook, rng)


def test_monte_carlo_distortion_through_pipeline():
    P.pin_mc_distortion(quantize, codebook, rng)


def test_attention_special_cases():
    P.pin_attention_special(attention)


def test_sparse_v_interval():
    P.pin_sparse_v(attention)


def test_rotated_domain_equals_original_domain():
    P.pin_rotated_domain(attention, quantize, codebook, rng)


def test_oracle_package_exports():
    assert {"rng", "rotation", "codebook", "quantize", "attention"} <= set(dir(oracle))


def test_masked_sparse_sum():
    P.pin_masked_sum(attention)


def test_prefill_causal_attention():
    P.pin_prefill(attention)

