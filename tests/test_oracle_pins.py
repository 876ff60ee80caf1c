"""Pins for the FP64 oracle against facts the pages and the mathematics fix (CPU only).

Each test would fail on a plausible slip in the oracle: a dropped surrogate term, the value mean in
place of the value sum, a missing 1/sqrt(d), a transposed proxy, the wrong sign of the Sol-Attn2
first-order correction, an off-by-one in the partial block, or a reversed threshold comparison.
"""
import math

import numpy as np
import pytest
import torch

from oracle import sol_attn_oracle as orc

D = 128
S = 1.0 / math.sqrt(D)


def dense_attention(q, k, v):
    """Textbook softmax attention through torch's SDPA (FP64, CPU); BTHD in and out."""
    qt, kt, vt = (torch.as_tensor(x, dtype=torch.float64).permute(0, 2, 1, 3) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)
    return o.permute(0, 2, 1, 3).numpy()


def rand_qkv(B, N, H, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return tuple(scale * g.standard_normal((B, N, H, D)) for _ in range(3))


# ---------------------------------------------------------------- dense limits (Eq. (2), M = 0)

@pytest.mark.parametrize("N", [64, 200, 256])
@pytest.mark.parametrize("entry", ["sol_attn", "sol_attn2"])
def test_sink_over_everything_is_dense_attention(N, entry):
    q, k, v = rand_qkv(1, N, 2, seed=N)
    fn = getattr(orc, entry)
    out = fn(q, k, v, tau=1.0, sink_start=0, sink_tokens=N)["out"]
    np.testing.assert_allclose(out, dense_attention(q, k, v), rtol=0, atol=1e-12)


@pytest.mark.parametrize("entry", ["sol_attn", "sol_attn2"])
def test_very_negative_tau_is_dense_attention(entry):
    q, k, v = rand_qkv(2, 300, 1, seed=7)
    r = getattr(orc, entry)(q, k, v, tau=-1e9)
    assert r["mask"].all()
    np.testing.assert_allclose(r["out"], dense_attention(q, k, v), rtol=0, atol=1e-12)


# ------------------------------------------------- surrogate exactness when a block's keys agree

def _sink_plus_identical_keys(N, H, seed):
    """Random q, v; keys random in blocks 0-1 (made exact by a sink), one shared key elsewhere."""
    g = np.random.default_rng(seed)
    q = g.standard_normal((1, N, H, D))
    v = g.standard_normal((1, N, H, D))
    k = np.empty((1, N, H, D))
    k[:, :128] = g.standard_normal((1, 128, H, D))
    k[:, 128:] = g.standard_normal((1, 1, H, D))
    return q, k, v


@pytest.mark.parametrize("N", [448, 460])   # 7 blocks, and 8 blocks with a partial 12-token tail
@pytest.mark.parametrize("entry", ["sol_attn", "sol_attn2"])
def test_identical_unselected_keys_make_the_approximation_exact(N, entry):
    """Taylor remainder (section 3.2) vanishes when k_u = Kbar_j; for Sol-Attn2 mu_a = k* gives
    Zhat_i = n e^{q_i.k*/sqrt d} and Uhat_i = Zhat_i * mean(v) exactly (first-order correction)."""
    q, k, v = _sink_plus_identical_keys(N, 2, seed=N)
    r = getattr(orc, entry)(q, k, v, tau=1e9, sink_start=0, sink_tokens=128)
    assert not r["mask"].all()            # the approximation really is in use
    np.testing.assert_allclose(r["out"], dense_attention(q, k, v), rtol=0, atol=1e-11)


def test_sol_attn_differs_from_dense_when_keys_vary():
    q, k, v = rand_qkv(1, 512, 1, seed=3)
    out = orc.sol_attn(q, k, v, tau=1.0)["out"]
    assert np.abs(out - dense_attention(q, k, v)).max() > 1e-4


# ------------------------------------------------------- approximation error bound (appendix)

def test_surrogate_error_bound_and_jensen():
    """0 <= D - D~ <= 1/2 e^{a+eta} sum delta_u^2 and |N - N~| <= e^{a+eta} sum |delta_u| |v_u|,
    a = s q.Kbar_j, delta_u = s q.(k_u - Kbar_j), eta = max_u |delta_u| (reading of eta)."""
    g = np.random.default_rng(11)
    for n in (64, 24):
        kb = 0.5 * g.standard_normal((n, D))
        vb = g.standard_normal((n, D))
        qr = g.standard_normal((16, D))
        Dt, Nt = orc.surrogate_terms(qr, kb.mean(axis=0), vb.sum(axis=0), n)
        a = S * qr @ kb.mean(axis=0)
        delta = S * qr @ (kb - kb.mean(axis=0)).T
        eta = np.abs(delta).max(axis=1)
        Dx = np.exp(S * qr @ kb.T).sum(axis=1)
        Nx = np.exp(S * qr @ kb.T) @ vb
        gap = Dx - Dt
        assert (gap >= -1e-12 * Dx).all()
        assert (gap <= 0.5 * np.exp(a + eta) * (delta**2).sum(axis=1) * (1 + 1e-12)).all()
        bound = np.exp(a + eta) * (np.abs(delta) * np.linalg.norm(vb, axis=1)[None, :]).sum(axis=1)
        assert (np.linalg.norm(Nx - Nt, axis=1) <= bound * (1 + 1e-12)).all()


# ----------------------------------------------------------------- threshold closed form (Eq. (5))

def test_threshold_definition_equals_covariance_form():
    g = np.random.default_rng(5)
    Nb = 37
    Qbar = g.standard_normal((Nb, D)) + 0.3
    Kbar = g.standard_normal((Nb, D)) - 0.2
    shat = orc.proxy_scores(Qbar, Kbar)
    mu, sigma, thr = orc.threshold(shat, tau=1.3)
    mK = Kbar.mean(axis=0)
    C = Kbar.T @ Kbar / Nb
    mu5 = S * Qbar @ mK
    var5 = S * S * np.einsum("id,de,ie->i", Qbar, C, Qbar) - mu5**2
    np.testing.assert_allclose(mu, mu5, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sigma**2, var5, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(thr, mu5 + 1.3 * np.sqrt(var5), rtol=1e-9)
    # the proxy is Qbar_i . Kbar_j, not its transpose
    assert shat[2, 5] == pytest.approx(S * Qbar[2] @ Kbar[5])


# ------------------------------------------------------------------------- routing rule pieces

def test_sink_blocks_by_hand():
    N = 200   # blocks [0,64) [64,128) [128,192) [192,200)
    f = lambda s, t: list(np.nonzero(orc.sink_block_flags(N, s, t))[0])
    assert f(0, 10) == [0]
    assert f(-1, 10) == [2, 3]           # suffix [190, 200)
    assert f(-1, 8) == [3]               # suffix [192, 200)
    assert f(64, 65) == [1, 2]           # interior [64, 129)
    assert f(150, 1000) == [2, 3]        # clipped at N
    assert f(0, 0) == [] and f(5, -3) == []
    assert f(0, 200) == [0, 1, 2, 3]


def test_huge_tau_keeps_only_adjacent_and_sink_blocks():
    q, k, _ = rand_qkv(1, 640, 1, seed=2)
    r = orc.routing(q, k, tau=1e9, sink_start=-1, sink_tokens=70)
    Nb = 10
    i = np.arange(Nb)
    expect = (np.abs(i[:, None] - i[None, :]) <= 1)
    expect[:, [8, 9]] = True             # suffix [570, 640) overlaps blocks 8 and 9
    assert (r["mask"][0, 0] == expect).all()


def test_threshold_direction_and_strict_ties():
    Nb = 8
    Qbar = np.zeros((Nb, D))
    Qbar[0, 0] = 1.0
    Kbar = np.zeros((Nb, D))
    Kbar[5, 0] = 10.0                     # block 5 has the largest proxy for query block 0
    Kbar[6, 0] = -10.0                    # block 6 the smallest
    shat = orc.proxy_scores(Qbar, Kbar)
    _, _, thr = orc.threshold(shat, tau=1.0)
    m = orc.exact_mask(shat, thr, np.zeros(Nb, bool))
    assert m[0, 5] and not m[0, 6] and not m[0, 3]
    # rows whose proxies are all equal have sigma = 0, tau_i = s_ij: nothing is strictly above
    assert m[3].sum() == 3 and m[3, 2] and m[3, 3] and m[3, 4]


def test_threshold_density_near_gaussian_calibration():
    """For near-Gaussian proxies the threshold-only density is close to 1 - Phi(beta)."""
    from scipy.stats import norm

    q, k, _ = rand_qkv(1, 8192, 4, seed=9)
    r = orc.routing(q, k, tau=1.0)
    above = r["shat"].astype(np.float32) > r["thresh"].astype(np.float32)[..., None]
    assert abs(above.mean() - (1 - norm.cdf(1.0))) < 0.02


# ------------------------------------------------------------------------- hand-expanded sums

def _hand_case():
    """N = 192 (3 blocks), H = 1. Queries (c + eps_r) e1; keys of blocks 0, 1: gamma e1; block 2:
    half (beta + alpha) e1, half (beta - alpha) e1 (interleaved). With tau huge, query block 0
    treats block 2 as unselected and query block 2 treats block 0 as unselected."""
    c, gamma, beta, alpha = 2.0, 0.5, 1.5, 0.7
    g = np.random.default_rng(17)
    N = 192
    eps = 0.3 * g.standard_normal(N)
    q = np.zeros((1, N, 1, D))
    q[0, :, 0, 0] = c + eps
    k = np.zeros((1, N, 1, D))
    k[0, :128, 0, 0] = gamma
    upper = np.arange(64) % 2 == 0
    k[0, 128:, 0, 0] = np.where(upper, beta + alpha, beta - alpha)
    v = g.standard_normal((1, N, 1, D))
    return dict(c=c, gamma=gamma, beta=beta, alpha=alpha, eps=eps, q=q, k=k, v=v, upper=upper)


def test_hand_expanded_sol_attn():
    h = _hand_case()
    r = orc.sol_attn(h["q"], h["k"], h["v"], tau=1e6)
    assert r["mask"][0, 0].tolist() == [[True, True, False], [True, True, True], [False, True, True]]
    v = h["v"][0, :, 0]
    for row in (0, 17, 63):           # query block 0: exact blocks 0, 1; block 2 is a surrogate
        x = h["c"] + h["eps"][row]
        we = math.exp(S * x * h["gamma"])
        ws = math.exp(S * x * h["beta"])   # Kbar_2 = beta e1
        expect = (we * v[:128].sum(0) + ws * v[128:].sum(0)) / (128 * we + 64 * ws)
        np.testing.assert_allclose(r["out"][0, row, 0], expect, rtol=1e-11, atol=1e-14)
    for row in (130, 191):            # query block 2: block 0 is a surrogate with Kbar_0 = gamma e1
        x = h["c"] + h["eps"][row]
        w0 = math.exp(S * x * h["gamma"])
        w2 = np.exp(S * x * h["k"][0, 128:, 0, 0])
        expect = (w0 * v[:128].sum(0) + w2 @ v[128:]) / (128 * w0 + w2.sum())
        np.testing.assert_allclose(r["out"][0, row, 0], expect, rtol=1e-11, atol=1e-14)


def test_hand_expanded_sol_attn2():
    h = _hand_case()
    r = orc.sol_attn2(h["q"], h["k"], h["v"], tau=1e6)
    v = h["v"][0, :, 0]
    eps = h["eps"]
    up = h["upper"]
    kg = {1: h["beta"] + h["alpha"], 0: h["beta"] - h["alpha"]}
    vg = {1: v[128:][up].mean(0), 0: v[128:][~up].mean(0)}
    for row in (0, 31, 32, 63):       # anchors 0 and 1 of query block 0; the tail is block 2
        a = row // 32
        xa = h["c"] + eps[32 * a: 32 * a + 32].mean()           # q_bar_a . e1
        w = {g: 32 * math.exp(S * xa * kg[g]) for g in (0, 1)}
        Z = w[0] + w[1]
        mu = (w[0] * kg[0] + w[1] * kg[1]) / Z
        nu = (w[0] * vg[0] + w[1] * vg[1]) / Z
        x = h["c"] + eps[row]
        delta = S * (x - xa) * mu
        Zhat = Z * math.exp(delta)
        we = math.exp(S * x * h["gamma"])
        expect = (we * v[:128].sum(0) + Zhat * nu) / (128 * we + Zhat)
        np.testing.assert_allclose(r["out"][0, row, 0], expect, rtol=1e-11, atol=1e-14)


# ---------------------------------------------------------------- Sol-Attn2 split direction

def _direction_case():
    """N = 192 (3 blocks), H = 1, in the e1-e2-e3 space.  Anchor bases (tokens 32a .. 32a + 31):
    (1, 2, 0), (1, 0, 0) | (1, -1, 0), (1, -1, 0) | (1, 0, 3), (1, 0, 3), plus +-0.25 e1 alternating
    inside each anchor (zero mean, so every anchor mean is its base).  The mean query is then
    u = (1, 0, 1), while query block 0's mean is (1, 1, 0), query block 2's is (1, 0, 3), anchor 0's
    is (1, 2, 0) and the keys' mean points elsewhere again: each candidate direction splits the tail
    blocks differently.  Tail blocks (tau huge: only |i - j| <= 1 is exact):
      key block 2 (tail of query block 0): 16 x P = (1, 0, 1) (projection on u: 2), 8 x M = (-2, 0, -2)
        (-4), 20 x (1, 0, -1) and 20 x (0, 1, 0) (both 0, exactly the block mean's projection);
      key block 0 (tail of query block 2): 12 x A = (2, 1, 0) (2), 8 x (0, 0, -3) (-3), 44 x (0, 2, 0) (0).
    Types are interleaved by a seeded permutation; values are random."""
    g = np.random.default_rng(29)
    N = 192
    q = np.zeros((1, N, 1, D))
    bases = [(1, 2, 0), (1, 0, 0), (1, -1, 0), (1, -1, 0), (1, 0, 3), (1, 0, 3)]
    for a, base in enumerate(bases):
        q[0, 32 * a: 32 * a + 32, 0, :3] = base
    eps = np.where(np.arange(N) % 2 == 0, 0.25, -0.25)
    q[0, :, 0, 0] += eps
    k = np.zeros((1, N, 1, D))
    blk2 = [(1, 0, 1)] * 16 + [(-2, 0, -2)] * 8 + [(1, 0, -1)] * 20 + [(0, 1, 0)] * 20
    blk0 = [(2, 1, 0)] * 12 + [(0, 0, -3)] * 8 + [(0, 2, 0)] * 44
    p2, p0 = g.permutation(64), g.permutation(64)
    k[0, 128:, 0, :3] = np.array(blk2, float)[p2]
    k[0, :64, 0, :3] = np.array(blk0, float)[p0]
    k[0, 64:128, 0, :3] = 0.5 * g.standard_normal((64, 3))
    upper2 = p2 < 16          # the P keys: the only keys of block 2 strictly above the split
    upper0 = p0 < 12          # the A keys of block 0
    v = g.standard_normal((1, N, 1, D))
    return dict(q=q, k=k, v=v, eps=eps, bases=np.array(bases, float), upper={2: upper2, 0: upper0})


def test_hand_expanded_sol_attn2_split_direction():
    """[Sol2] "Routing and complementary approximation": each unselected block splits into two groups
    by key projection on the mean-query direction (reading R10: the mean of all queries of the
    head; keys strictly above the block mean's projection form group 1).  The groups of both tail
    blocks are written out by hand from the construction, and the outputs of rows of both tail
    query blocks are expanded from them.  The key mean, a query block's or an anchor's mean, or
    -u would each group the keys differently (and the tied keys pin the side ties fall on)."""
    h = _direction_case()
    r = orc.sol_attn2(h["q"], h["k"], h["v"], tau=1e6)
    assert r["mask"][0, 0].tolist() == [[True, True, False], [True, True, True], [False, True, True]]
    assert r["group_counts"][0, 0, 2].tolist() == [48, 16]
    assert r["group_counts"][0, 0, 0].tolist() == [52, 12]
    q, k, v = h["q"][0, :, 0], h["k"][0, :, 0], h["v"][0, :, 0]
    for qi, tail, exact in ((0, 2, slice(0, 128)), (2, 0, slice(64, 192))):
        kb, vb = k[64 * tail: 64 * tail + 64], v[64 * tail: 64 * tail + 64]
        up = h["upper"][tail]
        groups = [(int((~up).sum()), kb[~up].mean(0), vb[~up].mean(0)), (int(up.sum()), kb[up].mean(0), vb[up].mean(0))]
        for row in (64 * qi, 64 * qi + 1, 64 * qi + 33, 64 * qi + 62):
            qa = np.zeros(D)
            qa[:3] = h["bases"][row // 32]
            w = [n * math.exp(S * float(qa @ kg)) for n, kg, _ in groups]
            Z = sum(w)
            mu = sum(wi * kg for wi, (_, kg, _) in zip(w, groups)) / Z
            nu = sum(wi * vg for wi, (_, _, vg) in zip(w, groups)) / Z
            Zhat = Z * math.exp(S * float((q[row] - qa) @ mu))
            we = np.exp(S * (k[exact] @ q[row]))
            expect = (we @ v[exact] + Zhat * nu) / (we.sum() + Zhat)
            np.testing.assert_allclose(r["out"][0, row, 0], expect, rtol=1e-11, atol=1e-14)


# ------------------------------------------------------------------------- mask override (parity)

@pytest.mark.parametrize("entry", ["sol_attn", "sol_attn2"])
def test_mask_override_evaluates_the_given_exact_sets(entry):
    """The override used by the GPU parity rule: the oracle's own mask reproduces its result, and an
    all-exact mask gives textbook softmax attention (Eq. (2) with every block selected), whatever
    the routing decided."""
    q, k, v = rand_qkv(1, 300, 2, seed=41)
    fn = getattr(orc, entry)
    r = fn(q, k, v, 1.0)
    assert not r["mask"].all()
    np.testing.assert_array_equal(fn(q, k, v, 1.0, mask_override=r["mask"])["out"], r["out"])
    dense = fn(q, k, v, 1.0, mask_override=np.ones_like(r["mask"]))
    np.testing.assert_allclose(dense["out"], dense_attention(q, k, v), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(dense["mask"], r["mask"])      # the routing is still reported


# ---------------------------------------------------------------------------- Sol-Attn2 groups

def test_group_counts_preserve_block_mass():
    g = np.random.default_rng(23)
    N = 200
    kb = g.standard_normal((N, D))
    vb = g.standard_normal((N, D))
    u = g.standard_normal(D)
    counts, kg, vg = orc.key_groups(kb, vb, u)
    assert (counts.sum(axis=1) == orc.block_counts(N)).all()
    for j in range(orc.num_blocks(N)):
        a, b = orc.block_range(j, N)
        np.testing.assert_allclose(counts[j] @ kg[j], kb[a:b].sum(0), atol=1e-10)
        np.testing.assert_allclose(counts[j] @ vg[j], vb[a:b].sum(0), atol=1e-10)
        proj = kb[a:b] @ u
        assert counts[j, 1] == int((proj > proj.mean()).sum())


# ------------------------------------------------------------------- accuracy claim (ablation)

def test_surrogate_reduces_error_against_dense():
    """Section 4.5, "Effect of Approximate Correction": with identical masks, adding the surrogate
    lowers the relative l2 error to dense attention compared with exact-only sparse attention."""
    from block_sparse_attention_sum_b200.inputs import GridSpec, grf_qkv

    q, k, v = (t.double().numpy() for t in grf_qkv(1, 2, GridSpec(4, 16, 32), seed_base=77))
    r = orc.sol_attn(q, k, v, tau=1.0)
    dense = dense_attention(q, k, v)
    N = q.shape[1]
    tok_mask = np.repeat(np.repeat(r["mask"], 64, axis=2), 64, axis=3)[:, :, :N, :N]
    qt, kt, vt = (torch.as_tensor(x).permute(0, 2, 1, 3) for x in (q, k, v))
    exact_only = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=torch.as_tensor(tok_mask)).permute(0, 2, 1, 3).numpy()
    rel = lambda x: np.linalg.norm(x - dense) / np.linalg.norm(dense)
    assert orc.realised_sparsity(r["mask"]) > 0.5
    assert rel(r["out"]) < rel(exact_only)


# ------------------------------------------------------------- diagonal threshold estimator

def test_diagonal_estimator_equals_exact_when_key_covariance_is_diagonal():
    """Appendix "Diagonal threshold estimator": with key-block means whose centred deviations have
    orthogonal channel columns, the covariance is diagonal and the estimator is exact."""
    g = np.random.default_rng(31)
    Nb = 160
    U, _ = np.linalg.qr(g.standard_normal((Nb, D)))          # orthonormal columns
    U -= U.mean(axis=0)                                       # centre ...
    U, _ = np.linalg.qr(U)                                    # ... and re-orthonormalise
    assert np.abs(U.mean(axis=0)).max() < 1e-12
    Kbar = 0.7 + U * g.uniform(0.5, 3.0, D)[None, :]
    Qbar = g.standard_normal((40, D))
    mu_e, sig_e, thr_e = orc.threshold(orc.proxy_scores(Qbar, Kbar), 1.1)
    mu_d, sig_d, thr_d = orc.threshold_diag(Qbar, Kbar, 1.1)
    np.testing.assert_allclose(mu_d, mu_e, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(sig_d, sig_e, rtol=1e-9)
    np.testing.assert_allclose(thr_d, thr_e, rtol=1e-9, atol=1e-12)


def test_diagonal_estimator_drops_channel_correlation():
    """With perfectly correlated channels the diagonal variance differs from the exact one by the
    off-diagonal terms, and equals the hand-computed sum of per-channel variances."""
    Nb = 50
    a = np.linspace(-1, 1, Nb)
    Kbar = np.zeros((Nb, D))
    Kbar[:, 0] = a
    Kbar[:, 1] = a                                            # channel 1 copies channel 0
    Qbar = np.zeros((1, D))
    Qbar[0, 0] = Qbar[0, 1] = 1.0
    _, sig_d, _ = orc.threshold_diag(Qbar, Kbar, 0.0)
    _, sig_e, _ = orc.threshold(orc.proxy_scores(Qbar, Kbar), 0.0)
    va = a.var()
    assert sig_d[0] == pytest.approx(S * np.sqrt(2 * va), rel=1e-12)
    assert sig_e[0] == pytest.approx(S * np.sqrt(4 * va), rel=1e-12)


# ---------------------------------------------------- several sink ranges and dense text rows (R16, R17)

def test_several_sink_ranges_hand_computed():
    # N = 1000: blocks of 64 tokens, the last one (960..999) partial.  Tokens 100..129 touch blocks
    # 1 and 2; token 700 lies in block 10; 990..1039 clips to 990..999 in block 15; the suffix of 5
    # tokens (995..999) is block 15 again.
    flags = orc.sink_block_flags(1000, -1, 5, extra_sinks=[(100, 30), (700, 1), (990, 50)])
    assert sorted(np.nonzero(flags)[0].tolist()) == [1, 2, 10, 15]
    assert not orc.sink_block_flags(1000, -1, 0, extra_sinks=[(5, 0)]).any()


def test_extra_sinks_force_exact_columns_for_every_row():
    q, k, _ = rand_qkv(1, 640, 1, seed=11)
    r = orc.routing(q, k, tau=3.0, sink_start=0, sink_tokens=64, extra_sinks=[(300, 10), (600, 40)])
    m = r["mask"][0, 0]
    assert m[:, [0, 4, 9]].all()     # blocks 0 (0..63), 4 (256..319), 9 (576..639)


def test_dense_rows_match_library_attention():
    q, k, v = rand_qkv(1, 300, 2, seed=5)
    out = orc.dense_rows(q, k, v, 70, 81)
    ref = dense_attention(q, k, v)
    np.testing.assert_allclose(out[:, 70:151], ref[:, 70:151], rtol=0, atol=1e-12)
    assert np.isnan(out[:, :70]).all() and np.isnan(out[:, 151:]).all()
    suf = orc.dense_rows(q, k, v, -1, 20)
    np.testing.assert_allclose(suf[:, 280:], ref[:, 280:], rtol=0, atol=1e-12)


def test_dense_rows_with_identical_keys_average_the_values():
    q, k, v = rand_qkv(1, 130, 1, seed=6)
    k[:] = k[:, :1]
    out = orc.dense_rows(q, k, v, 0, 130)
    np.testing.assert_allclose(out[0, :, 0], np.broadcast_to(v[0, :, 0].mean(axis=0), (130, D)), rtol=0, atol=1e-12)
