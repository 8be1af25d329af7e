"""The CPU oracle against its pins (published vectors, hand-worked examples,
closed forms, laws and library special cases). No GPU needed."""
import pytest

import oracle
from tests import oracle_pins as P


def test_splitmix64_published_vectors():
    P.check_splitmix64_vectors(oracle)


def test_table_moments():
    P.check_table_moments(oracle)


def test_table_laws_ks():
    P.check_table_laws(oracle)


def test_table_prefix_layout():
    P.check_table_prefix(oracle)


def test_bins_worked_examples():
    P.check_bins_worked(oracle)


def test_varlen_spans_match_block_ends():
    P.check_varlen_spans_from_blocks(oracle)


def test_blocks_contiguous():
    P.check_contiguous_blocks(oracle)


def test_interior_block_lengths():
    P.check_block_lengths(oracle)


def test_boundary_bits_identity():
    P.check_boundary_identity(oracle)


@pytest.mark.slow
def test_expectation_identity_monte_carlo():
    P.check_expectation_identity(oracle)


@pytest.mark.slow
def test_theorem_2_1_rate():
    P.check_thm21_rate(oracle)


def test_bmax_law():
    P.check_bmax_law(oracle)


def test_bmax_loglog_growth():
    P.check_bmax_loglog(oracle)


def test_tiny_attention_worked_example():
    P.check_tiny_attention(oracle)


def test_s1_is_per_bin_softmax():
    P.check_s1_per_bin_softmax(oracle)


def test_one_bin_is_dense_softmax():
    P.check_one_bin_dense(oracle)


def test_singleton_bins_give_v():
    P.check_singleton_bins(oracle)


def test_exact_alibi_is_additive_bias_softmax():
    P.check_exact_alibi_sdpa(oracle)


@pytest.mark.slow
def test_convergence_in_s():
    P.check_convergence(oracle)


def test_sampled_rows_and_gqa():
    P.check_rows_and_gqa(oracle)


def test_exact_alibi_multi_head_gqa():
    P.check_forward_exact_gqa(oracle)


def test_gradients_match_autograd_of_log_count_bias():
    P.check_grad_autograd(oracle)


def test_gradients_match_finite_differences():
    P.check_grad_finite_differences(oracle)


def test_gradients_of_singleton_bins():
    P.check_grad_singleton_bins(oracle)


def test_backward_gqa():
    P.check_backward_gqa(oracle)


def test_sampled_gradients_equal_full():
    P.check_grad_sampled_equals_full(oracle)
