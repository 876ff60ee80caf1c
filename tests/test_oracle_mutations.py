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


def _direction_key_mean(q_bh, k_bh):
    return k_bh.mean(axis=0)


def _direction_first_anchor(q_bh, k_bh):
    return q_bh[: orc.ANCHOR].mean(axis=0)


def _direction_flipped(q_bh, k_bh):
    return -q_bh.mean(axis=0)


_orig_key_groups = orc.key_groups


def _ties_upper(k_bh, v_bh, u):
    N = k_bh.shape[0]
    Nb = orc.num_blocks(N)
    counts, kg, vg = np.zeros((Nb, 2), np.int64), np.zeros((Nb, 2, orc.HEAD_DIM)), np.zeros((Nb, 2, orc.HEAD_DIM))
    for j in range(Nb):
        a, b = orc.block_range(j, N)
        proj = (k_bh[a:b] @ u).astype(np.float32)
        upper = proj >= np.float32(k_bh[a:b].mean(axis=0) @ u)
        for g, sel in ((0, ~upper), (1, upper)):
            counts[j, g] = int(sel.sum())
            if counts[j, g]:
                kg[j, g], vg[j, g] = k_bh[a:b][sel].mean(axis=0), v_bh[a:b][sel].mean(axis=0)
    return counts, kg, vg


def _groups_median_split(k_bh, v_bh, u):
    # equal halves (split at the median projection) instead of the block mean's projection
    N = k_bh.shape[0]
    Nb = orc.num_blocks(N)
    counts, kg, vg = np.zeros((Nb, 2), np.int64), np.zeros((Nb, 2, orc.HEAD_DIM)), np.zeros((Nb, 2, orc.HEAD_DIM))
    for j in range(Nb):
        a, b = orc.block_range(j, N)
        order = np.argsort(k_bh[a:b] @ u, kind="stable")
        half = (b - a) // 2
        for g, sel in ((0, order[:half]), (1, order[half:])):
            counts[j, g] = len(sel)
            if len(sel):
                kg[j, g], vg[j, g] = k_bh[a:b][sel].mean(axis=0), v_bh[a:b][sel].mean(axis=0)
    return counts, kg, vg


def _sol_attn2_per_query_block_direction(q, k, v, tau, sink_start=-1, sink_tokens=0, qblocks=None, heads=None,
                                         extra_sinks=()):
    # the reading the oracle rejects: every query block splits the keys on its own mean query
    B, N, H, _ = q.shape
    Nb = orc.num_blocks(N)
    sink = orc.sink_block_flags(N, sink_start, sink_tokens, extra_sinks)
    out = np.full((B, N, H, orc.HEAD_DIM), np.nan)
    masks = np.zeros((B, H, Nb, Nb), dtype=bool)
    group_counts = np.zeros((B, H, Nb, 2), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            q_bh, k_bh, v_bh = orc.head_slice(q, b, h), orc.head_slice(k, b, h), orc.head_slice(v, b, h)
            r = orc._routing_for_head(q_bh, k_bh, tau, sink)
            masks[b, h] = r["mask"]
            qbar_anchor = orc.block_means(q_bh, orc.ANCHOR)
            for i in range(Nb):
                lo, hi = orc.block_range(i, N)
                counts, kg, vg = orc.key_groups(k_bh, v_bh, q_bh[lo:hi].mean(axis=0))
                out[b, lo:hi, h] = orc.sol_attn2_rows(q_bh[lo:hi], lo, k_bh, v_bh, r["mask"][i], counts, kg, vg,
                                                      qbar_anchor)
            group_counts[b, h] = orc.key_groups(k_bh, v_bh, orc.group_direction(q_bh, k_bh))[0]
    return dict(out=out, mask=masks, group_counts=group_counts)


_orig_sol_attn = orc.sol_attn


def _override_ignored(q, k, v, tau, *args, mask_override=None, **kw):
    return _orig_sol_attn(q, k, v, tau, *args, **kw)


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
    ("group_direction", _direction_key_mean, pins.test_hand_expanded_sol_attn2_split_direction),
    ("group_direction", _direction_first_anchor, pins.test_hand_expanded_sol_attn2_split_direction),
    ("group_direction", _direction_flipped, pins.test_hand_expanded_sol_attn2_split_direction),
    ("key_groups", _ties_upper, pins.test_hand_expanded_sol_attn2_split_direction),
    ("key_groups", _groups_median_split, pins.test_hand_expanded_sol_attn2_split_direction),
    ("sol_attn2", _sol_attn2_per_query_block_direction, pins.test_hand_expanded_sol_attn2_split_direction),
    ("sol_attn", _override_ignored, lambda: pins.test_mask_override_evaluates_the_given_exact_sets("sol_attn")),
]


@pytest.mark.parametrize("name,broken,pin", CASES, ids=[f"{c[0]}-{i}" for i, c in enumerate(CASES)])
def test_planted_mistake_is_caught(monkeypatch, name, broken, pin):
    monkeypatch.setattr(orc, name, broken)
    with pytest.raises(AssertionError):
        pin()


# ---------------------------------------------------------------- FP8 + ExpCast reference
from oracle import fp8_oracle as f8  # noqa: E402
from tests import test_oracle_fp8 as fp8pins  # noqa: E402


def _decode_bias_8(code):
    c = np.asarray(code, dtype=np.int64)
    e, m = c >> 3, c & 7
    return np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * 2.0 ** (e - 8.0))


def _expcast_no_clip(u):
    return f8.e4m3_decode(np.maximum(np.round(8.0 * np.asarray(u, dtype=np.float64) + f8.EXPCAST_OFFSET), 0).astype(np.int64))


def _quantize_no_scale(x):
    x = np.asarray(x, dtype=np.float64)
    return f8.e4m3_round(x), 1.0


_orig_fp8_rows = f8.sol_attn_fp8_rows


def _fp8_surrogate_sums(q8_rows, k8_bh, v8_bh, mask_row, kbar8, vbar8, counts):
    return _orig_fp8_rows(q8_rows, k8_bh, v8_bh, mask_row, kbar8, vbar8 * counts[:, None], counts)


def _surrogate_one_key_scale(Kbar, Vhat, counts, v_amax):
    _, vbar8 = _orig_surrogate(Kbar, Vhat, counts, v_amax)
    return f8.quantize(Kbar)[0], vbar8


def _surrogate_sums_quantised(Kbar, Vhat, counts, v_amax):
    kbar8, _ = _orig_surrogate(Kbar, Vhat, counts, v_amax)
    return kbar8, f8.quantize_with_max(Vhat, v_amax)[0]


def _quantize_scale_first(x):
    # X / fl(max / 448): the order that rounds exact midpoints the wrong way
    x = np.asarray(x, dtype=np.float64)
    amax = float(np.abs(x).max())
    s = amax / 448.0 if amax > 0 else 1.0
    return s * f8.e4m3_round(x / s), s


_orig_surrogate = f8.surrogate_operands_fp8


def _sol2_fp8_tail_without_pivot(q8_rows, row0, k8_bh, v8_bh, mask_row, counts, kg, vg, qbar_anchor):
    # the tail mass added without the pivot's factor 2^-pivot
    import math as _m
    from oracle import sol_attn_oracle as _orc
    N = k8_bh.shape[0]
    ex = np.nonzero(mask_row)[0]
    un = np.nonzero(~mask_row)[0]
    tok = np.concatenate([np.arange(*_orc.block_range(j, N)) for j in ex])
    z = _orc.SCALE * (q8_rows @ k8_bh[tok].T)
    tc, tk, tv = counts[un].reshape(-1), kg[un].reshape(-1, 128), vg[un].reshape(-1, 128)
    keep = tc > 0
    out = np.empty_like(q8_rows)
    for r in range(q8_rows.shape[0]):
        a = (row0 + r) // _orc.ANCHOR
        logZ, mu_a, nu_a = _orc.anchor_tail(qbar_anchor[a], tc[keep], tk[keep], tv[keep])
        pivot = np.ceil(z[r].max() / _m.log(2.0)) - 8.0
        pz = f8.expcast(z[r] / _m.log(2.0) - pivot)
        zt = _m.exp(logZ + _orc.SCALE * ((q8_rows[r] - qbar_anchor[a]) @ mu_a)) if np.isfinite(logZ) else 0.0
        out[r] = (pz @ v8_bh[tok] + zt * nu_a) / (pz.sum() + zt)
    return out


FP8_CASES = [
    ("e4m3_decode", _decode_bias_8, fp8pins.test_e4m3_decode_matches_torch),
    ("expcast_code", lambda u: np.round(8.0 * np.asarray(u) + f8.EXPCAST_OFFSET).astype(np.int64),
     fp8pins.test_expcast_powers_of_two_and_error_bound),
    ("expcast", _expcast_no_clip, fp8pins.test_expcast_powers_of_two_and_error_bound),
    ("quantize", _quantize_no_scale, fp8pins.test_quantizer_extremes),
    ("quantize", _quantize_scale_first, fp8pins.test_quantizer_rounds_exact_midpoints_to_even),
    ("sol_attn_fp8_rows", _fp8_surrogate_sums, fp8pins.test_fp8_forward_with_zero_queries_averages_the_values),
    ("surrogate_operands_fp8", _surrogate_one_key_scale,
     fp8pins.test_surrogate_operands_are_quantised_like_keys_and_values),
    ("surrogate_operands_fp8", _surrogate_sums_quantised,
     fp8pins.test_surrogate_operands_are_quantised_like_keys_and_values),
    ("surrogate_operands_fp8", _surrogate_sums_quantised,
     fp8pins.test_fp8_forward_with_zero_queries_averages_the_values),
    ("sol_attn2_fp8_rows", _sol2_fp8_tail_without_pivot, fp8pins.test_fp8_sol2_with_zero_queries_averages_the_values),
]


@pytest.mark.parametrize("name,broken,pin", FP8_CASES, ids=[f"fp8-{c[0]}-{i}" for i, c in enumerate(FP8_CASES)])
def test_planted_fp8_mistake_is_caught(monkeypatch, name, broken, pin):
    monkeypatch.setattr(f8, name, broken)
    with pytest.raises(AssertionError):
        pin()
