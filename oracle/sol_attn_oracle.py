"""Plain FP64 CPU oracle for the Sol-Attn and Sol-Attn2 forward operators.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline
leg (including ``bench.py --impl reference``) may import or call this module.  The product path
(the CUDA library and its Python binding) never routes through it.  It shares no code with the
CUDA path: the only common dependency is the seeded input generator, which holds none of the
method's arithmetic.

Every step is written from the pages' definitions, in their order and notation, with FP64 values
(BF16 inputs widen exactly) and a library matmul / logsumexp as the only primitives.  There is no
tiling, fusion or reordering beyond what the definitions state.

Sources (page title, section / equation):

* [SolAttn]  "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly Attention
  Sparsification" (arXiv 2607.24027): Eq. (2) block-sparse attention, Eq. (3) pooled proxy scores,
  Eq. (4) threshold routing, Eq. (5) efficient threshold, Eq. (6) chunk proxies, section 3.2
  "Proxy-Score Reuse as Approximate Correction" (Taylor expansion, denominator D_i, token-to-block
  scores), "Hardware-Aligned Implementation" (pooled key KC and summed value VC), appendix
  "Threshold variance derivation" and "Approximation error".
* [Sol2]     "Sol-Attn2: Sparse Attention with Complementary Approximation" (draft), Method,
  "Routing and complementary approximation" (w_ag, Z_a, mu_a, nu_a, delta_i, o_i) and
  "How the outputs are combined" (alpha_i).
* [README]   Sol-Attn library README (NVlabs/Sana sparse_backends): "Core API" (BF16 BTHD,
  head dim 128, tau), "Exact KV sink" (prefix / suffix / interior sink at 64-token block
  granularity).
* [sdcpp]    stable-diffusion.cpp "Sol-Attn" documentation: adjacent blocks remain exact; K means
  and V sums for the approximate blocks; one shared online-softmax normaliser.

Readings where the pages are silent, ambiguous or garbled:

R1  Scale: s = 1/sqrt(128) on token logits, proxies, thresholds and surrogate logits ([Sol2] uses
    z = q.k/sqrt(d); the paper's Eqs. (1)-(3) print no scale).  The routing mask does not depend
    on it (tau * sigma scales with it); only the surrogate does.
R2  "N" in Eq. (5) is the number of key blocks Nb; every block, the partial last one included,
    has equal weight in mu_i and sigma_i.
R3  Threshold type "exact" (full covariance), the README default; evaluated here by its
    definition (mean and variance of the proxy row), which Eq. (5) restates.  Type "diag" follows
    the appendix's diagonal estimator (exact mean, diagonal of the key-mean covariance).
R4  Ties s_ij == tau_i are not exact (strict ">", Eq. (4)).
R5  Adjacent blocks: key blocks j with |i - j| <= 1 are always exact ([sdcpp]).
R6  Partial last block: means over its valid tokens, surrogate mass n_j (its token count).
R7  Surrogate numerator: exp(s q.Kbar_j) * Vhat_j with Vhat_j the block's value SUM
    ("summed value" in "Hardware-Aligned Implementation"); denominator n_j exp(s q.Kbar_j)
    (D_i, section 3.2, with B = n_j).  Both per query TOKEN (token-to-block scores).
R8  Sink with sink_start < 0: a suffix [N - sink_tokens, N) ("Omit" in the README table).
    sink_tokens <= 0: no sink.  The range is clipped to [0, N).
R9  Sol-Attn2 exact set E_i: the same threshold rule (tau), adjacency and sink.
R10 Sol-Attn2 "mean-query direction": one direction per (batch, head), u = mean of all queries.
    Key groups are query independent: group 1 = keys with k.u > Kbar_j.u, group 0 = the rest.
R11 Sol-Attn2 anchors: anchor a covers tokens [32a, 32a + 32) (clipped to N), q_bar_a is their
    mean, and its tail uses E of query block floor(a / 2).  Empty groups are skipped; an empty
    tail gives Zhat = 0.
R12 Sol-Attn2 does not add the Sol-Attn surrogate: the complementary tail replaces it.
R13 Routing decisions are taken on FP32-rounded proxy and threshold values (the precision the
    kernel decides in); the values themselves are computed in FP64.
R16 Several sink ranges (the README describes one contiguous range; texts split into segments need
    several): each range is applied as the README's sink, and a key block is exact if it overlaps
    any of them.
R17 Dense text rows ([README] "Exact KV sink": the sink does not make text query rows dense; an
    MMDiT integration should use dense attention for the valid text queries): plain softmax
    attention of those query tokens over all keys, o_r = sum_t e^{s q_r.k_t} v_t / sum_t e^{s q_r.k_t}.
"""
from __future__ import annotations

import math

import numpy as np

HEAD_DIM = 128
BLOCK = 64
ANCHOR = 32
SCALE = 1.0 / math.sqrt(HEAD_DIM)


# ----------------------------------------------------------------------------------------------
# inputs
# ----------------------------------------------------------------------------------------------

def to_f64(x) -> np.ndarray:
    """Widen a BF16 torch tensor, or any float array, to an FP64 numpy array (exact for BF16)."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def head_slice(x, b: int, h: int) -> np.ndarray:
    """[N, 128] FP64 rows of one (batch, head) of a BTHD tensor."""
    try:
        import torch

        if isinstance(x, torch.Tensor):
            return x[b, :, h, :].to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x[b, :, h, :], dtype=np.float64)


def num_blocks(N: int, size: int = BLOCK) -> int:
    return (N + size - 1) // size


def block_range(j: int, N: int, size: int = BLOCK) -> tuple[int, int]:
    return j * size, min(N, (j + 1) * size)


# ----------------------------------------------------------------------------------------------
# block summaries: [SolAttn] Eq. (3) (pooled Qbar, Kbar), "Hardware-Aligned Implementation"
# (pooled key KC[j] = Kbar_j, summed value VC[j] = Vhat_j); reading R6 for the partial block.
# ----------------------------------------------------------------------------------------------

def block_means(x: np.ndarray, size: int = BLOCK) -> np.ndarray:
    """Mean over the valid tokens of each ``size``-token block of an [N, d] array."""
    N = x.shape[0]
    return np.stack([x[a:b].mean(axis=0) for a, b in (block_range(j, N, size) for j in range(num_blocks(N, size)))])


def block_sums(x: np.ndarray) -> np.ndarray:
    N = x.shape[0]
    return np.stack([x[a:b].sum(axis=0) for a, b in (block_range(j, N) for j in range(num_blocks(N)))])


def block_counts(N: int) -> np.ndarray:
    return np.array([b - a for a, b in (block_range(j, N) for j in range(num_blocks(N)))], dtype=np.int64)


# ----------------------------------------------------------------------------------------------
# routing: [SolAttn] Eq. (3) proxies, Eq. (4) threshold, appendix "Threshold variance derivation"
# (first line: the definition of mu_i and sigma_i), README "Exact KV sink", [sdcpp] adjacency.
# ----------------------------------------------------------------------------------------------

def proxy_scores(Qbar: np.ndarray, Kbar: np.ndarray) -> np.ndarray:
    """s_hat[i, j] = s * Qbar_i . Kbar_j (Eq. (3) with reading R1)."""
    return SCALE * (Qbar @ Kbar.T)


def threshold(shat: np.ndarray, tau: float):
    """mu_i, sigma_i of row i of the proxy map by their definition; tau_i = mu_i + tau * sigma_i.

    The API's ``tau`` is the paper's beta (README: higher values select fewer blocks).
    """
    Nb = shat.shape[1]
    mu = shat.sum(axis=1) / Nb
    var = ((shat - mu[:, None]) ** 2).sum(axis=1) / Nb
    sigma = np.sqrt(var)
    return mu, sigma, mu + tau * sigma


def threshold_diag(Qbar: np.ndarray, Kbar: np.ndarray, tau: float):
    """Diagonal threshold estimator (appendix "Diagonal threshold estimator"): the mean mu_i is
    exact; the variance keeps only the diagonal of the key-mean covariance,
    v_K = mean_j Kbar_j * Kbar_j - mu_K * mu_K and sigma_i^2 = (Qbar_i * Qbar_i) . v_K (scaled by s^2,
    reading R1).  Returns mu, sigma, tau_i = mu_i + tau * sigma_i."""
    Nb = Kbar.shape[0]
    muK = Kbar.sum(axis=0) / Nb
    vK = (Kbar * Kbar).sum(axis=0) / Nb - muK * muK
    mu = SCALE * (Qbar @ muK)
    sigma = SCALE * np.sqrt(np.maximum((Qbar * Qbar) @ vK, 0.0))
    return mu, sigma, mu + tau * sigma


def sink_block_flags(N: int, sink_start: int, sink_tokens: int, extra_sinks=()) -> np.ndarray:
    """Key blocks that overlap an exact sink range (README "Exact KV sink"; readings R8, R16).

    ``extra_sinks``: further (start, tokens) ranges with start >= 0, each applied like the first."""
    Nb = num_blocks(N)
    flags = np.zeros(Nb, dtype=bool)
    for rs, rt in [(sink_start, sink_tokens)] + list(extra_sinks):
        if rt <= 0:
            continue
        start = rs if rs >= 0 else N - rt
        end = min(N, start + rt)
        start = max(0, start)
        for j in range(Nb):
            a, b = block_range(j, N)
            if a < end and b > start:
                flags[j] = True
    return flags


def exact_mask(shat: np.ndarray, thresh: np.ndarray, sink_flags: np.ndarray) -> np.ndarray:
    """E[i, j]: s_hat_ij > tau_i (decided on FP32-rounded values, R13), or |i-j| <= 1, or sink."""
    Nb = shat.shape[0]
    above = shat.astype(np.float32) > thresh.astype(np.float32)[:, None]
    idx = np.arange(Nb)
    adjacent = np.abs(idx[:, None] - idx[None, :]) <= 1
    return above | adjacent | sink_flags[None, :]


# ----------------------------------------------------------------------------------------------
# Sol-Attn output: [SolAttn] Eq. (2) for the exact blocks, section 3.2 proxy-score reuse for the
# rest (R7), one shared normaliser; M is only a common shift for numerical range.
# ----------------------------------------------------------------------------------------------

def surrogate_terms(q_rows: np.ndarray, Kbar_j: np.ndarray, Vhat_j: np.ndarray, n_j: int, shift=None):
    """Approximate denominator and numerator of one unselected block for each query row.

    D~ = n_j exp(s q.Kbar_j - shift), N~ = exp(s q.Kbar_j - shift) Vhat_j.
    """
    a = SCALE * (q_rows @ Kbar_j)
    if shift is None:
        shift = np.zeros_like(a)
    e = np.exp(a - shift)
    return n_j * e, e[:, None] * Vhat_j[None, :]


def sol_attn_rows(q_rows, k_bh, v_bh, mask_row, Kbar, Vhat, counts):
    """Outputs of the query rows of one query block (one (b, h)), given its exact-set row."""
    N = k_bh.shape[0]
    ex = np.nonzero(mask_row)[0]
    un = np.nonzero(~mask_row)[0]
    tok = np.concatenate([np.arange(*block_range(j, N)) for j in ex]) if len(ex) else np.zeros(0, np.int64)
    z = SCALE * (q_rows @ k_bh[tok].T)                                   # exact token logits
    a = SCALE * (q_rows @ Kbar[un].T)                                    # surrogate logits
    logmass = a + np.log(counts[un].astype(np.float64))[None, :]         # log(n_j e^a)
    M = np.full(q_rows.shape[0], -np.inf)
    if z.shape[1]:
        M = np.maximum(M, z.max(axis=1))
    if a.shape[1]:
        M = np.maximum(M, logmass.max(axis=1))
    pz = np.exp(z - M[:, None])
    pa = np.exp(a - M[:, None])
    den = pz.sum(axis=1) + (pa * counts[un][None, :]).sum(axis=1)
    num = pz @ v_bh[tok] + pa @ Vhat[un]
    return num / den[:, None]


def _routing_for_head(q_bh, k_bh, tau, sink_flags, thresh_type="exact"):
    N = q_bh.shape[0]
    Qbar = block_means(q_bh)
    Kbar = block_means(k_bh)
    shat = proxy_scores(Qbar, Kbar)
    if thresh_type == "diag":
        mu, sigma, thresh = threshold_diag(Qbar, Kbar, tau)
    else:
        mu, sigma, thresh = threshold(shat, tau)
    mask = exact_mask(shat, thresh, sink_flags)
    return dict(Qbar=Qbar, Kbar=Kbar, shat=shat, mu=mu, sigma=sigma, thresh=thresh, mask=mask,
                counts=block_counts(N))


def routing(q, k, tau: float, sink_start: int = -1, sink_tokens: int = 0, thresh_type: str = "exact",
            extra_sinks=()):
    """Per (b, h): proxies, mu, sigma, thresholds and exact masks. Returns a dict of stacked arrays."""
    B, N, H, _ = q.shape
    sink = sink_block_flags(N, sink_start, sink_tokens, extra_sinks)
    per = [[_routing_for_head(head_slice(q, b, h), head_slice(k, b, h), tau, sink, thresh_type) for h in range(H)]
           for b in range(B)]
    keys = ["shat", "mu", "sigma", "thresh", "mask"]
    return {key: np.stack([np.stack([per[b][h][key] for h in range(H)]) for b in range(B)]) for key in keys}


def _row_subset(N, qblocks):
    Nb = num_blocks(N)
    return range(Nb) if qblocks is None else qblocks


def sol_attn(q, k, v, tau: float, sink_start: int = -1, sink_tokens: int = 0, qblocks=None, heads=None,
             thresh_type: str = "exact", extra_sinks=(), mask_override=None):
    """Sol-Attn forward. Returns dict with ``out`` (FP64 [B, N, H, 128]; NaN for rows not computed),
    ``mask`` [B, H, Nb, Nb], ``shat``, ``thresh``.

    ``qblocks``: optional iterable of query-block indices to evaluate (all heads); ``heads``:
    optional iterable of (b, h) pairs.  Summaries and thresholds are always computed in full.
    ``mask_override``: optional bool [B, H, Nb, Nb] exact sets to evaluate the outputs with instead
    of this routing's (the parity rule for pairs whose proxy lies within the margin of its
    threshold, where a kernel's rounding may decide the other way); ``mask`` still reports the
    oracle's own routing.
    """
    B, N, H, _ = q.shape
    Nb = num_blocks(N)
    sink = sink_block_flags(N, sink_start, sink_tokens, extra_sinks)
    out = np.full((B, N, H, HEAD_DIM), np.nan)
    masks = np.zeros((B, H, Nb, Nb), dtype=bool)
    shats = np.zeros((B, H, Nb, Nb))
    threshs = np.zeros((B, H, Nb))
    pairs = [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)
    for b, h in pairs:
        q_bh, k_bh, v_bh = head_slice(q, b, h), head_slice(k, b, h), head_slice(v, b, h)
        r = _routing_for_head(q_bh, k_bh, tau, sink, thresh_type)
        Vhat = block_sums(v_bh)
        masks[b, h], shats[b, h], threshs[b, h] = r["mask"], r["shat"], r["thresh"]
        use = r["mask"] if mask_override is None else np.asarray(mask_override[b, h], dtype=bool)
        for i in _row_subset(N, qblocks):
            lo, hi = block_range(i, N)
            out[b, lo:hi, h] = sol_attn_rows(q_bh[lo:hi], k_bh, v_bh, use[i], r["Kbar"], Vhat, r["counts"])
    return dict(out=out, mask=masks, shat=shats, thresh=threshs)


# ----------------------------------------------------------------------------------------------
# Sol-Attn2 complementary tail: [Sol2] "Routing and complementary approximation", readings R9-R12.
# ----------------------------------------------------------------------------------------------

def group_direction(q_bh: np.ndarray, k_bh: np.ndarray) -> np.ndarray:
    """The direction the keys are split on ([Sol2] "Routing and complementary approximation": the
    mean-query direction), per reading R10: the mean of all queries of the (batch, head), one
    direction shared by every anchor and query block.  ``k_bh`` is unused (it is part of the
    signature so that readings based on the keys can be compared in the tests)."""
    return q_bh.mean(axis=0)


def key_groups(k_bh: np.ndarray, v_bh: np.ndarray, u: np.ndarray):
    """Two content groups per key block, split by the key projection on direction u (R10).

    Returns counts [Nb, 2], kbar_g [Nb, 2, 128], vbar_g [Nb, 2, 128] (zeros for empty groups).
    """
    N = k_bh.shape[0]
    Nb = num_blocks(N)
    counts = np.zeros((Nb, 2), dtype=np.int64)
    kg = np.zeros((Nb, 2, HEAD_DIM))
    vg = np.zeros((Nb, 2, HEAD_DIM))
    for j in range(Nb):
        a, b = block_range(j, N)
        kb, vb = k_bh[a:b], v_bh[a:b]
        proj = (kb @ u).astype(np.float32)
        cut = np.float32(kb.mean(axis=0) @ u)
        upper = proj > cut
        for g, sel in ((0, ~upper), (1, upper)):
            counts[j, g] = int(sel.sum())
            if counts[j, g]:
                kg[j, g] = kb[sel].mean(axis=0)
                vg[j, g] = vb[sel].mean(axis=0)
    return counts, kg, vg


def anchor_tail(qbar_a: np.ndarray, tail_counts, tail_k, tail_v):
    """log Z_a, mu_a, nu_a over the tail groups of one anchor (w_ag = n_g exp(s qbar_a.kbar_g))."""
    if len(tail_counts) == 0:
        return -np.inf, np.zeros(HEAD_DIM), np.zeros(HEAD_DIM)
    logw = np.log(tail_counts.astype(np.float64)) + SCALE * (tail_k @ qbar_a)
    c = logw.max()
    w = np.exp(logw - c)
    Z = w.sum()
    return c + math.log(Z), (w @ tail_k) / Z, (w @ tail_v) / Z


def sol_attn2_rows(q_rows, row0, k_bh, v_bh, mask_row, counts, kg, vg, qbar_anchor):
    """Outputs of the query rows [row0, row0 + len) of one query block under Sol-Attn2."""
    N = k_bh.shape[0]
    ex = np.nonzero(mask_row)[0]
    un = np.nonzero(~mask_row)[0]
    tok = np.concatenate([np.arange(*block_range(j, N)) for j in ex]) if len(ex) else np.zeros(0, np.int64)
    z = SCALE * (q_rows @ k_bh[tok].T)
    t_counts = counts[un].reshape(-1)
    t_k = kg[un].reshape(-1, HEAD_DIM)
    t_v = vg[un].reshape(-1, HEAD_DIM)
    keep = t_counts > 0
    t_counts, t_k, t_v = t_counts[keep], t_k[keep], t_v[keep]
    out = np.empty_like(q_rows)
    for r in range(q_rows.shape[0]):
        a = (row0 + r) // ANCHOR
        logZ, mu_a, nu_a = anchor_tail(qbar_anchor[a], t_counts, t_k, t_v)
        if np.isfinite(logZ):
            delta = SCALE * ((q_rows[r] - qbar_anchor[a]) @ mu_a)
            logZhat = logZ + delta
        else:
            logZhat = -np.inf
        zr = z[r]
        M = max(zr.max() if zr.size else -np.inf, logZhat)
        pz = np.exp(zr - M)
        zt = math.exp(logZhat - M) if np.isfinite(logZhat) else 0.0
        out[r] = (pz @ v_bh[tok] + zt * nu_a) / (pz.sum() + zt)
    return out


def sol_attn2(q, k, v, tau: float, sink_start: int = -1, sink_tokens: int = 0, qblocks=None, heads=None,
              extra_sinks=(), mask_override=None):
    """Sol-Attn2 forward (complementary tail). Same return convention as :func:`sol_attn`, plus
    ``group_counts`` [B, H, Nb, 2]: n_g of the two key groups of every block (group 1 = the keys
    whose projection on the direction lies strictly above the block mean's).  ``mask_override`` as in
    :func:`sol_attn`."""
    B, N, H, _ = q.shape
    Nb = num_blocks(N)
    sink = sink_block_flags(N, sink_start, sink_tokens, extra_sinks)
    out = np.full((B, N, H, HEAD_DIM), np.nan)
    masks = np.zeros((B, H, Nb, Nb), dtype=bool)
    group_counts = np.zeros((B, H, Nb, 2), dtype=np.int64)
    pairs = [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)
    for b, h in pairs:
        q_bh, k_bh, v_bh = head_slice(q, b, h), head_slice(k, b, h), head_slice(v, b, h)
        r = _routing_for_head(q_bh, k_bh, tau, sink)
        masks[b, h] = r["mask"]
        counts, kg, vg = key_groups(k_bh, v_bh, group_direction(q_bh, k_bh))
        group_counts[b, h] = counts
        qbar_anchor = block_means(q_bh, ANCHOR)
        use = r["mask"] if mask_override is None else np.asarray(mask_override[b, h], dtype=bool)
        for i in _row_subset(N, qblocks):
            lo, hi = block_range(i, N)
            out[b, lo:hi, h] = sol_attn2_rows(q_bh[lo:hi], lo, k_bh, v_bh, use[i], counts, kg, vg, qbar_anchor)
    return dict(out=out, mask=masks, group_counts=group_counts)


def dense_rows(q, k, v, q_start: int, q_tokens: int):
    """Dense attention of the query tokens [q_start, q_start + q_tokens) over all keys (R17);
    ``q_start < 0`` selects the suffix.  Returns FP64 [B, N, H, 128], NaN outside the rows."""
    B, N, H, _ = q.shape
    out = np.full((B, N, H, HEAD_DIM), np.nan)
    if q_tokens <= 0:
        return out
    r0 = q_start if q_start >= 0 else N - q_tokens
    r1 = min(N, r0 + q_tokens)
    r0 = max(0, r0)
    for b in range(B):
        for h in range(H):
            q_bh, k_bh, v_bh = head_slice(q, b, h), head_slice(k, b, h), head_slice(v, b, h)
            z = SCALE * (q_bh[r0:r1] @ k_bh.T)
            z -= z.max(axis=1, keepdims=True)
            e = np.exp(z)
            out[b, r0:r1, h] = (e @ v_bh) / e.sum(axis=1, keepdims=True)
    return out


def realised_sparsity(mask: np.ndarray) -> float:
    """Fraction of (query-block, key-block) pairs that are not exact."""
    return 1.0 - float(mask.sum()) / mask.size


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round FP64 values to BF16 (nearest even) and return them as FP64."""
    f = np.asarray(x, dtype=np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    rounded = ((bits + 0x7FFF + ((bits >> 16) & 1)) >> 16) << 16
    out = rounded.astype(np.uint32).view(np.float32).astype(np.float64)
    return np.where(np.isfinite(f), out, f.astype(np.float64))
