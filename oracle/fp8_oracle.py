"""FP64 reference for the FP8 (E4M3) + ExpCast variant of the Sol-Attn forward.

TEST INFRASTRUCTURE ONLY, like ``sol_attn_oracle``: only the tests (and the bench's CPU legs) may
import it; the product path never does.  It shares no code with the CUDA path.

Source: "Sol-Attn2: Sparse Attention with Complementary Approximation", section "FP8 quantization
and ExpCast":

* Q and K are quantised with one E4M3 scale per 64-token block, V with one scale per head: for a
  nonzero block X, s_X = max|X| / 448, X_8 = FP8_E4M3(X / s_X), X ~= s_X X_8.
* QK and PV use the FP8 operands with FP32 accumulation; the scales restore the magnitudes.
* ExpCast turns a base-2 score directly into an E4M3 probability byte: with a shared online pivot m,
  u = (s - m) log2 e, c(u) = clip_[0,120](RNE(8u + 55.65)), p(u) = decode_E4M3(c(u)) ~= 2^u.  The same
  decoded weights enter the PV product and the denominator.

Readings:

R18 Both products of the shared softmax take FP8 operands (the section gives FP8 operands to QK and
    PV and keeps the mass of the compressed keys by a bias added to their scores): the exact
    branch's tokens as above, and the
    surrogate's compressed keys and values under the same rules - the block means Kbar_j quantised
    as a key array (one scale per 64 consecutive compressed keys of a head), the value means
    Vbar_j = Vhat_j / n_j with the head's V scale (|Vbar| <= max |V|, so they stay in range).  A
    surrogate block's logit is q8 . Kbar8_j / sqrt(d) plus the additive bias ln n_j, its value
    Vbar8_j per unit of that mass.  Routing (block means, thresholds, masks) stays as in the BF16
    path, computed from the original inputs.
R19 ExpCast gives every weight of the shared softmax, exact tokens and surrogate blocks alike (the
    surrogate's log-mass ln n_j is part of its score, as in the BF16 path); numerator and denominator
    use the same decoded weights.  The pivot is an integer in base 2: ExpCast is not invariant under
    fractional shifts of u, but for an integer shift k the code moves by exactly 8k (one E4M3
    binade), so weights coded against any integer pivot agree up to the factor 2^-k except below
    2^-6 of the pivot (subnormal codes and the clip at 0).  The code range [0, 120] spans
    u in [-6.96, 8.04]: a pivot at the maximum would leave half of it unused and drop every weight
    below 2^-7 of the maximum, so the reference takes the pivot ceil(row max) - 8 in base 2
    (u <= 8, the largest weight coded 112..120), the range an online pivot moved only when the
    running maximum exceeds it by more than 8 keeps.  An online pass differs in one respect: a weight
    coded before the pivot moved keeps its code, while this final pivot clips every weight more than
    ~7 binades below it (about 15 binades below the row maximum).  The two agree whenever no such
    weight exists, which covers ordinary inputs; a row whose maximum jumps by 14 binades after many
    small scores (keys scaled by 0.25, then by 3) differs by ~6e-3 relative l2.
R20 An all-zero quantisation block keeps scale 1 and zero codes.
R22 The quotient X / s_X is the exact real number 448 X / max|X| rounded to E4M3 (nearest, ties to
    even); it is evaluated in that form (exact products for BF16 inputs), not as X / fl(s_X).
R21 Sol-Attn2 under FP8: the exact branch as above (E4M3 operands, ExpCast weights against the
    integer pivot ceil(max exact score / ln 2) - 8); the complementary tail's Z_a, mu_a, nu_a are
    those of the BF16 path (computed from the original inputs: the tail is not a product of the
    shared softmax); delta_i takes the dequantised query s_Q Q8_i, and Zhat_i enters the shared
    denominator with its exact exponential relative to the same pivot (one term per row, not a
    probability byte of a PV product).
"""
from __future__ import annotations

import math

import numpy as np

from oracle import sol_attn_oracle as orc

E4M3_MAX = 448.0
EXPCAST_OFFSET = 55.65
EXPCAST_MAX_CODE = 120


def e4m3_round(x) -> np.ndarray:
    """Round to the nearest E4M3 value (ties to even), saturating at +-448.

    E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; normal values (1 + m/8) 2^(e-7)
    for e = 1..15 (largest finite 1.75 * 2^8 = 448), subnormals m 2^-9."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))           # binade, at least the smallest normal one
    step = 2.0 ** (e - 3)                                      # 3 mantissa bits (2^-9 for subnormals)
    r = np.round(a / step) * step                              # numpy rounds half to even
    return np.sign(x) * np.minimum(r, E4M3_MAX)


def e4m3_decode(code) -> np.ndarray:
    """Value of non-negative E4M3 codes 0..126 (bit pattern 0 eeee mmm)."""
    c = np.asarray(code, dtype=np.int64)
    e, m = c >> 3, c & 7
    return np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))


def expcast_code(u) -> np.ndarray:
    """c(u) = clip_[0,120](RNE(8u + 55.65))."""
    return np.clip(np.round(8.0 * np.asarray(u, dtype=np.float64) + EXPCAST_OFFSET), 0, EXPCAST_MAX_CODE).astype(np.int64)


def expcast(u) -> np.ndarray:
    """p(u) = decode_E4M3(c(u)) ~= 2^u."""
    return e4m3_decode(expcast_code(u))


def quantize(x) -> tuple[np.ndarray, float]:
    """One E4M3 scale for the whole array: (s_X X_8 as FP64, s_X).

    X / s_X is evaluated as 448 X / max|X|, the same real number: for inputs with few mantissa bits
    (BF16) the product is exact and the quotient exact whenever it is representable, so a value
    exactly halfway between two E4M3 numbers stays halfway and rounds to even, as the definition
    asks.  X / fl(max|X| / 448) carries the rounding of s_X and can land one unit off the midpoint
    (R22)."""
    x = np.asarray(x, dtype=np.float64)
    amax = float(np.abs(x).max()) if x.size else 0.0
    return quantize_with_max(x, amax)


def quantize_with_max(x, amax: float) -> tuple[np.ndarray, float]:
    """(s X_8, s) with s = amax / 448 for an array whose scale comes from amax (the max of a larger
    set, e.g. the head's V for the value means); amax = 0 gives scale 1 and zero codes (R20)."""
    x = np.asarray(x, dtype=np.float64)
    if amax <= 0:
        return np.zeros_like(x), 1.0
    s = amax / E4M3_MAX
    return s * e4m3_round(x * E4M3_MAX / amax), s


def quantize_blocks(x_bh: np.ndarray, block: int = orc.BLOCK) -> np.ndarray:
    """Per 64-token block of one head's [N, 128] rows (the last block partial): dequantised E4M3."""
    out = np.empty_like(np.asarray(x_bh, dtype=np.float64))
    for j in range(orc.num_blocks(x_bh.shape[0])):
        a, b = orc.block_range(j, x_bh.shape[0])
        out[a:b] = quantize(x_bh[a:b])[0]
    return out


def sol_attn_fp8_rows(q8_rows, k8_bh, v8_bh, mask_row, kbar8, vbar8, counts):
    """Outputs of one query block's rows under the FP8 path.

    Exact tokens: logits from the dequantised E4M3 operands (FP64 here; FP32 accumulation in the
    kernel), values from the dequantised V.  Surrogate blocks: logits q8 . Kbar8_j / sqrt(d) plus
    ln n_j, values Vbar8_j per unit of mass (R18).  Every weight is ExpCast of its base-2 score
    against the integer pivot ceil(row max / ln 2) - 8 (R19)."""
    N = k8_bh.shape[0]
    ex = np.nonzero(mask_row)[0]
    un = np.nonzero(~mask_row)[0]
    tok = np.concatenate([np.arange(*orc.block_range(j, N)) for j in ex]) if len(ex) else np.zeros(0, np.int64)
    z = orc.SCALE * (q8_rows @ k8_bh[tok].T)
    logmass = orc.SCALE * (q8_rows @ kbar8[un].T) + np.log(counts[un].astype(np.float64))[None, :]
    M = np.full(q8_rows.shape[0], -np.inf)
    if z.shape[1]:
        M = np.maximum(M, z.max(axis=1))
    if logmass.shape[1]:
        M = np.maximum(M, logmass.max(axis=1))
    pivot = np.ceil(M / math.log(2.0)) - 8.0                            # integer base-2 pivot
    pz = expcast(z / math.log(2.0) - pivot[:, None])
    pa = expcast(logmass / math.log(2.0) - pivot[:, None])
    num = pz @ v8_bh[tok] + pa @ vbar8[un]
    den = pz.sum(axis=1) + pa.sum(axis=1)
    return num / den[:, None]


def surrogate_operands_fp8(Kbar, Vhat, counts, v_amax: float):
    """E4M3 compressed keys and values of one head (R18): Kbar per 64 consecutive block means,
    Vbar = Vhat / n with the head's V scale (v_amax = max |V| of the head)."""
    kbar8 = quantize_blocks(Kbar)
    vbar = Vhat / counts[:, None]
    return kbar8, quantize_with_max(vbar, v_amax)[0]


def sol_attn_fp8(q, k, v, tau: float, sink_start: int = -1, sink_tokens: int = 0, qblocks=None, mask_override=None):
    """FP8 + ExpCast Sol-Attn forward.  Returns dict with ``out`` (FP64, NaN for rows not computed)
    and ``mask`` (the routing of the BF16 path, R18).  ``mask_override`` as in the BF16 oracle."""
    B, N, H, _ = q.shape
    Nb = orc.num_blocks(N)
    sink = orc.sink_block_flags(N, sink_start, sink_tokens)
    out = np.full((B, N, H, orc.HEAD_DIM), np.nan)
    masks = np.zeros((B, H, Nb, Nb), dtype=bool)
    for b in range(B):
        for h in range(H):
            q_bh, k_bh, v_bh = orc.head_slice(q, b, h), orc.head_slice(k, b, h), orc.head_slice(v, b, h)
            r = orc._routing_for_head(q_bh, k_bh, tau, sink)
            masks[b, h] = r["mask"]
            q8, k8 = quantize_blocks(q_bh), quantize_blocks(k_bh)
            v8 = quantize(v_bh)[0]
            kbar8, vbar8 = surrogate_operands_fp8(r["Kbar"], orc.block_sums(v_bh), r["counts"], float(np.abs(v_bh).max()))
            use = r["mask"] if mask_override is None else np.asarray(mask_override[b, h], dtype=bool)
            for i in (range(Nb) if qblocks is None else qblocks):
                lo, hi = orc.block_range(i, N)
                out[b, lo:hi, h] = sol_attn_fp8_rows(q8[lo:hi], k8, v8, use[i], kbar8, vbar8, r["counts"])
    return dict(out=out, mask=masks)


def sol_attn2_fp8_rows(q8_rows, row0, k8_bh, v8_bh, mask_row, counts, kg, vg, qbar_anchor):
    """Outputs of the query rows [row0, row0 + len) of one query block under FP8 Sol-Attn2 (R21)."""
    N = k8_bh.shape[0]
    ex = np.nonzero(mask_row)[0]
    un = np.nonzero(~mask_row)[0]
    tok = np.concatenate([np.arange(*orc.block_range(j, N)) for j in ex]) if len(ex) else np.zeros(0, np.int64)
    z = orc.SCALE * (q8_rows @ k8_bh[tok].T)
    t_counts = counts[un].reshape(-1)
    t_k = kg[un].reshape(-1, orc.HEAD_DIM)
    t_v = vg[un].reshape(-1, orc.HEAD_DIM)
    keep = t_counts > 0
    t_counts, t_k, t_v = t_counts[keep], t_k[keep], t_v[keep]
    out = np.empty_like(q8_rows)
    for r in range(q8_rows.shape[0]):
        a = (row0 + r) // orc.ANCHOR
        logZ, mu_a, nu_a = orc.anchor_tail(qbar_anchor[a], t_counts, t_k, t_v)
        zr = z[r]
        pivot = (np.ceil(zr.max() / math.log(2.0)) - 8.0) if zr.size else 0.0
        pz = expcast(zr / math.log(2.0) - pivot)
        if np.isfinite(logZ):
            delta = orc.SCALE * ((q8_rows[r] - qbar_anchor[a]) @ mu_a)
            zt = math.exp(logZ + delta - pivot * math.log(2.0))
        else:
            zt = 0.0
        out[r] = (pz @ v8_bh[tok] + zt * nu_a) / (pz.sum() + zt)
    return out


def sol_attn2_fp8(q, k, v, tau: float, sink_start: int = -1, sink_tokens: int = 0, qblocks=None, mask_override=None):
    """FP8 + ExpCast Sol-Attn2 forward (R21).  Same return convention as :func:`sol_attn_fp8`."""
    B, N, H, _ = q.shape
    Nb = orc.num_blocks(N)
    sink = orc.sink_block_flags(N, sink_start, sink_tokens)
    out = np.full((B, N, H, orc.HEAD_DIM), np.nan)
    masks = np.zeros((B, H, Nb, Nb), dtype=bool)
    for b in range(B):
        for h in range(H):
            q_bh, k_bh, v_bh = orc.head_slice(q, b, h), orc.head_slice(k, b, h), orc.head_slice(v, b, h)
            r = orc._routing_for_head(q_bh, k_bh, tau, sink)
            masks[b, h] = r["mask"]
            counts, kg, vg = orc.key_groups(k_bh, v_bh, orc.group_direction(q_bh, k_bh))
            qbar_anchor = orc.block_means(q_bh, orc.ANCHOR)
            q8, k8 = quantize_blocks(q_bh), quantize_blocks(k_bh)
            v8 = quantize(v_bh)[0]
            use = r["mask"] if mask_override is None else np.asarray(mask_override[b, h], dtype=bool)
            for i in (range(Nb) if qblocks is None else qblocks):
                lo, hi = orc.block_range(i, N)
                out[b, lo:hi, h] = sol_attn2_fp8_rows(q8[lo:hi], lo, k8, v8, use[i], counts, kg, vg, qbar_anchor)
    return dict(out=out, mask=masks)
