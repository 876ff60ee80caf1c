"""Comparison helpers for the GPU-vs-oracle parity tests.

Routing decisions: the GPU mask must equal the oracle's bit for bit, except for pairs whose proxy
margin |s_ij - tau_i| is within MARGIN (scaled units); forced pairs (adjacent, sink) must always be
set.  Outputs: compared element by element within MAX_ABS and REL_L2 on every computed row: where a
pair inside the margin was decided the other way, the oracle is re-run for that query block with the
GPU's exact sets (``with_gpu_mask``), so no row is left out of the comparison.
"""
import inspect

import numpy as np

MARGIN = 1e-3
MAX_ABS = 2e-2
REL_L2 = 5e-3


def check_mask(gpu_mask, ref, sink_flags=None):
    """Returns the boolean [B, H, Nb] array of query-block rows whose masks differ."""
    gm = np.asarray(gpu_mask).astype(bool)
    om = ref["mask"]
    assert gm.shape == om.shape, (gm.shape, om.shape)
    Nb = om.shape[-1]
    i = np.arange(Nb)
    adjacent = np.abs(i[:, None] - i[None, :]) <= 1
    assert gm[..., adjacent].all(), "adjacent blocks must be exact"
    if sink_flags is not None and sink_flags.any():
        assert gm[..., sink_flags].all(), "sink blocks must be exact"
    diff = gm != om
    if diff.any():
        margin = np.abs(ref["shat"] - ref["thresh"][..., None])
        bad = diff & (margin > MARGIN)
        assert not bad.any(), f"{int(bad.sum())} mask mismatches outside the {MARGIN} margin"
    return diff.any(axis=-1)


def with_gpu_mask(fn, args, gpu_mask, skip, ref_out, **kwargs):
    """The oracle's outputs with the rows of every query block in ``skip`` (the [B, H, Nb] rows
    whose masks differ, all within the margin as check_mask has verified) replaced by the oracle
    ``fn(*args, **kwargs)`` re-run with the GPU's exact sets as ``mask_override``."""
    skip = np.asarray(skip, dtype=bool)
    if not skip.any():
        return ref_out
    bs, hs, rows = np.nonzero(skip)
    kw = dict(kwargs, qblocks=sorted(set(rows.tolist())), mask_override=np.asarray(gpu_mask).astype(bool))
    if "heads" in inspect.signature(fn).parameters:
        kw["heads"] = sorted({(int(b), int(h)) for b, h in zip(bs, hs)})
    redo = fn(*args, **kw)["out"]
    out = np.array(ref_out, copy=True)
    N = out.shape[1]
    for b, h, i in zip(bs, hs, rows):
        lo, hi = 64 * i, min(N, 64 * i + 64)
        out[b, lo:hi, h] = redo[b, lo:hi, h]
    return out


def compare_outputs(gpu_out, ref_out, N, skip_rows=None, qblocks=None, max_abs_tol=MAX_ABS, rel_l2_tol=REL_L2):
    """gpu_out: BF16/float tensor [B, N, H, 128]; ref_out: FP64 oracle (NaN where not computed)."""
    g = np.asarray(gpu_out, dtype=np.float64)
    r = np.asarray(ref_out)
    B, _, H, _ = r.shape
    sel = ~np.isnan(r[..., 0])                  # [B, N, H]
    if skip_rows is not None:
        Nb = skip_rows.shape[-1]
        tok_blk = np.minimum(np.arange(N) // 64, Nb - 1)
        skip_tok = skip_rows[:, :, tok_blk].transpose(0, 2, 1)   # [B, N, H]
        sel &= ~skip_tok
    assert sel.any(), "nothing to compare"
    d = g[sel] - r[sel]
    max_abs = float(np.abs(d).max())
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(r[sel]), 1e-30))
    assert np.isfinite(g[sel]).all(), "non-finite GPU output"
    assert max_abs <= max_abs_tol, f"max abs error {max_abs:.3e} > {max_abs_tol}"
    assert rel <= rel_l2_tol, f"relative l2 error {rel:.3e} > {rel_l2_tol}"
    return max_abs, rel, int(sel.sum())


def model_rows_with_agreeing_masks(qd, kd, q, k, tau, ss=-1, st=0):
    """Token rows whose query block has the same exact set on the GPU router as in the reference's
    routing, which the FP32 model of the FP8 kernels uses (a pair within the proxy margin may
    differ).  qd, kd: the device tensors; q, k: the same on the CPU."""
    from block_sparse_attention_sum_b200 import sol_attn as sa
    from oracle import sol_attn_oracle as orc

    N = q.shape[1]
    gmask, _ = sa.debug_route(qd, kd, tau, ss, st)
    full = orc.routing(q, k, tau, ss, st)
    skip = check_mask(gmask.cpu().numpy(), full, orc.sink_block_flags(N, ss, st))
    rows = ~np.repeat(skip[0, 0], 64)[:N]
    assert rows.mean() >= 0.9
    return rows
