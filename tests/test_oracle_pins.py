"""The oracle against what the pages and the mathematics fix (CPU only)."""
import pytest

from tests import oracle_checks as C


def test_yarn_closed_form_golden():
    assert C.check_yarn_golden() < 1e-12


def test_rope_matches_qwen2_rotary_embedding():
    # transformers computes its angles in float32: loose bound, still O(1) on a
    # sign, pairing or frequency mistake
    assert C.check_rope_vs_transformers() < 2e-4


def test_rope_is_complex_rotation():
    assert C.check_rope_complex() < 1e-12


def test_rope_depends_on_relative_position():
    assert C.check_rope_relative() < 1e-10


def test_dca_logits_brute_force():
    assert C.check_dca_brute_force() < 1e-10


def test_dca_relative_positions_within_trained_range_and_exact_near():
    assert C.check_dca_invariants()


def test_short_sequence_is_causal_rope_attention():
    assert C.check_short_equals_causal_rope() < 1e-10


def test_v_ones_gives_ones():
    assert C.check_v_ones() < 1e-12


def test_full_budget_is_dense():
    assert C.check_full_budget_is_dense() < 1e-12


def test_causality():
    assert C.check_causal() < 1e-12


def test_lse_merge_identity():
    assert C.check_lse_merge() < 1e-12


def test_estimator_mass_and_lse():
    assert C.check_estimator_mass() < 1e-5


def test_estimator_brute_force():
    assert C.check_estimator_brute_force() < 1e-6


def test_topk_properties_with_ties():
    assert C.check_topk_properties()


def test_forced_local_diagonals():
    assert C.check_force_local()


def test_block_mask_brute_force():
    assert C.check_mask_brute_force()


def test_attended_set_enumeration():
    assert C.check_attended_set()


def test_recall_identity_and_full_budget():
    assert C.check_recall() < 1e-12


def test_equal_cost_chunks_fixture_and_invariants():
    assert C.check_equal_cost_chunks() > 200


def test_decode_row_brute_force():
    assert C.check_decode_row() < 1e-10


def test_key_order_invariance():
    assert C.check_key_order_invariance() < 1e-12


def test_residual_verticals_complete_the_attended_set():
    assert C.check_residual_verticals()


def test_fixed_prefill_chunks():
    assert C.check_fixed_chunks()
