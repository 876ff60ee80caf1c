"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin catches each one.

Each case swaps one oracle function or constant for a broken variant, runs a pin from
test_oracle_pins, and expects it to fail.  This shows the pins constrain every step of the oracle.
"""
import numpy as np
import pytest

from oracle import sol_attn_oracle as orc
from tests import test_oracle_pins as pins


def _value_means_not_sums(x):
    N = x.shape[0]
    return np.stack([x[a:b].mean(axis=0) for a, b in (orc.block_range(j, N) for j in range(orc.num_blocks(N)))])


def _full_block_counts(N):
    return np.full(orc.num_blocks(N), orc.BLOCK, dtype=np.int64)


def _transposed_proxy(Qbar, Kbar):
    return orc.SCALE * (Kbar @ Qbar.T)


def _sample_variance(shat, tau):
    mu = shat.mean(axis=1)
    sigma = shat.std(axis=1, ddof=1)
    return mu, sigma, mu + tau * sigma


def _reversed_comparison(shat, thresh, sink_flags):
    Nb = shat.shape[0]
    idx = np.arange(Nb)
    return (shat < thresh[:, None]) | (np.abs(idx[:, None] - idx[None, :]) <= 1) | sink_flags[None, :]


def _no_adjacency(shat, thresh, sink_flags):
    return (shat.astype(np.float32) > thresh.astype(np.float32)[:, None]) | sink_flags[None, :]


_orig_anchor_tail = orc.anchor_tail


def _flipped_mu(qbar_a, tail_counts, tail_k, tail_v):
    logZ, mu, nu = _orig_anchor_tail(qbar_a, tail_counts, tail_k, tail_v)
    return logZ, -mu, nu


def _mu_is_nu(qbar_a, tail_counts, tail_k, tail_v):
    logZ, mu, nu = _orig_anchor_tail(qbar_a, tail_counts, tail_k, tail_v)
    return logZ, nu, nu


def _unweighted_groups(qbar_a, tail_counts, tail_k, tail_v):
    return _orig_anchor_tail(qbar_a, np.ones_like(tail_counts), tail_k, tail_v)


def _suffix_off_by_one(N, sink_start, sink_tokens):
    return _orig_sink(N, sink_start if sink_start >= 0 else N - sink_tokens - 1, sink_tokens)


_orig_sink = orc.sink_block_flags


def _extra_sinks_ignored(N, sink_start, sink_tokens, extra_sinks=()):
    return _orig_sink(N, sink_start, sink_tokens)


_orig_dense = orc.dense_rows


def _dense_rows_one_short(q, k, v, q_start, q_tokens):
    return _orig_dense(q, k, v, q_start, q_tokens - 1)


def _dense_rows_unscaled(q, k, v, q_start, q_tokens):
    return _orig_dense(q / orc.SCALE, k, v, q_start, q_tokens)


_orig_diag = orc.threshold_diag


def _diag_without_mean(Qbar, Kbar, tau):
    mu, sigma, thresh = _orig_diag(Qbar, Kbar, tau)
    return 0.0 * mu, sigma, tau * sigma


CASES = [
    ("block_sums", _value_means_not_sums,
     lambda: pins.test_identical_unselected_keys_make_the_approximation_exact(448, "sol_attn")),
    ("block_counts", _full_block_counts,
     lambda: pins.test_identical_unselected_keys_make_the_approximation_exact(460, "sol_attn")),
    ("proxy_scores", _transposed_proxy, pins.test_threshold_definition_equals_covariance_form),
    ("threshold", _sample_variance, pins.test_threshold_definition_equals_covariance_form),
    ("exact_mask", _reversed_comparison, pins.test_threshold_direction_and_strict_ties),
    ("exact_mask", _no_adjacency, pins.test_huge_tau_keeps_only_adjacent_and_sink_blocks),
    ("anchor_tail", _flipped_mu,
     lambda: pins.test_identical_unselected_keys_make_the_approximation_exact(448, "sol_attn2")),
    ("anchor_tail", _mu_is_nu, pins.test_hand_expanded_sol_attn2),
    ("anchor_tail", _unweighted_groups, pins.test_hand_expanded_sol_attn2),
    ("sink_block_flags", _suffix_off_by_one, pins.test_sink_blocks_by_hand),
    ("SCALE", 1.0, lambda: pins.test_sink_over_everything_is_dense_attention(200, "sol_attn")),
    ("SCALE", 2.0 * orc.SCALE, pins.test_hand_expanded_sol_attn),
    ("sink_block_flags", _extra_sinks_ignored, pins.test_several_sink_ranges_hand_computed),
    ("dense_rows", _dense_rows_one_short, pins.test_dense_rows_match_library_attention),
    ("dense_rows", _dense_rows_unscaled, pins.test_dense_rows_match_library_attention),
    ("threshold_diag", _diag_without_mean, pins.test_diagonal_estimator_equals_exact_when_key_covariance_is_diagonal),
]


@pytest.mark.parametrize("name,broken,pin", CASES, ids=[f"{c[0]}-{i}" for i, c in enumerate(CASES)])
def test_planted_mistake_is_caught(monkeypatch, name, broken, pin):
    monkeypatch.setattr(orc, name, broken)
    with pytest.raises(AssertionError):
        pin()
