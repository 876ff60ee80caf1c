"""GPU parity: the CUDA library (through its C ABI) against the FP64 oracle on the same inputs.

Routing: masks bit-exact outside the 1e-3 proxy margin, forced blocks always exact, thresholds to
FP32 rounding.  Outputs: max-abs <= 2e-2 and relative l2 <= 5e-3 against the oracle, element by
element, on every query block whose mask row agrees (all of them unless a near-tie flipped).
Small and ragged shapes run in full; the 32K-128K workloads compare 16 seeded query blocks per head
(all heads) plus the full routing mask, in the launch configuration the bench times.
"""
import zlib

import numpy as np
import pytest
import torch

from block_sparse_attention_sum_b200 import sol_attn as sa
from block_sparse_attention_sum_b200.inputs import iid_qkv
from block_sparse_attention_sum_b200.workloads import WORKLOADS
from oracle import sol_attn_oracle as orc
from tests.parity import check_mask, compare_outputs, with_gpu_mask

pytestmark = pytest.mark.gpu


def _to_gpu(*ts):
    return [t.cuda() for t in ts]


def _run(entry, q, k, v, tau, sink_start, sink_tokens):
    qd, kd, vd = _to_gpu(q, k, v)
    fn = sa.sol_attn_fwd if entry == "sol_attn" else sa.sol_attn2_fwd
    out = fn(qd, kd, vd, tau, sink_start, sink_tokens)
    torch.cuda.synchronize()
    assert sa.get_device_status() == 0
    return out.float().cpu().numpy(), (qd, kd, vd)


SMALL = [
    # name, B, N, H, tau, sink_start, sink_tokens
    ("n64", 1, 64, 1, 1.0, -1, 0),
    ("n65_b2_h3", 2, 65, 3, 1.0, -1, 0),
    ("n127", 1, 127, 2, 0.5, -1, 0),
    ("n129", 1, 129, 2, 1.0, -1, 0),
    ("n200_suffix_sink", 1, 200, 2, 1.0, -1, 10),
    ("n1000_b2", 2, 1000, 2, 1.0, -1, 0),
    ("n1000_interior_sink", 1, 1000, 2, 1.5, 300, 200),
    ("n2048_dense_sink", 1, 2048, 2, 1.0, 0, 2048),
    ("n4000_high_tau", 1, 4000, 2, 3.0, -1, 0),
    ("n4096_low_tau", 1, 4096, 1, -0.5, -1, 0),
]


def _small_inputs(name, B, N, H):
    return iid_qkv(B, N, H, seed=zlib.crc32(name.encode()) % 1000)


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
@pytest.mark.parametrize("entry", ["sol_attn", "sol_attn2"])
def test_small_and_ragged(case, entry):
    name, B, N, H, tau, ss, st = case
    q, k, v = _small_inputs(name, B, N, H)
    ref = getattr(orc, entry)(q, k, v, tau, ss, st)
    gout, (qd, kd, _) = _run(entry, q, k, v, tau, ss, st)
    gmask, gthr = sa.debug_route(qd, kd, tau, ss, st)
    full = orc.routing(q, k, tau, ss, st)
    ref.update(shat=full["shat"], thresh=full["thresh"])
    gm = gmask.cpu().numpy()
    skip = check_mask(gm, ref, orc.sink_block_flags(N, ss, st))
    compare_outputs(gout, with_gpu_mask(getattr(orc, entry), (q, k, v, tau, ss, st), gm, skip, ref["out"]), N)


@pytest.mark.parametrize("name", ["tiny", "wan"])
@pytest.mark.parametrize("entry", ["sol_attn", "sol_attn2"])
def test_named_workloads_in_full(name, entry):
    w = WORKLOADS[name]
    q, k, v = w.make_inputs("cpu")
    tau = w.resolved_tau()
    ref = getattr(orc, entry)(q, k, v, tau, w.sink_start, w.sink_tokens)
    full = orc.routing(q, k, tau, w.sink_start, w.sink_tokens)
    ref.update(shat=full["shat"], thresh=full["thresh"])
    gout, (qd, kd, _) = _run(entry, q, k, v, tau, w.sink_start, w.sink_tokens)
    gmask, gthr = sa.debug_route(qd, kd, tau, w.sink_start, w.sink_tokens)
    gm = gmask.cpu().numpy()
    skip = check_mask(gm, ref)
    assert skip.mean() <= 0.01
    np.testing.assert_allclose(gthr.cpu().numpy(), full["thresh"], rtol=1e-5, atol=2e-6)
    args = (q, k, v, tau, w.sink_start, w.sink_tokens)
    compare_outputs(gout, with_gpu_mask(getattr(orc, entry), args, gm, skip, ref["out"]), w.N)


LARGE = ["s32k_80", "s32k_85", "s32k_90", "s64k", "s128k", "sol2_64k"]


@pytest.mark.parametrize("name", LARGE)
def test_large_workloads_sampled(name):
    w = WORKLOADS[name]
    q, k, v = w.make_inputs("cpu")
    tau = w.resolved_tau()
    Nb = orc.num_blocks(w.N)
    sample = sorted(np.random.default_rng(7).choice(Nb, size=16, replace=False).tolist())
    fn = getattr(orc, w.entry)
    ref = fn(q, k, v, tau, w.sink_start, w.sink_tokens, qblocks=sample)
    full = orc.routing(q, k, tau, w.sink_start, w.sink_tokens)
    ref.update(shat=full["shat"], thresh=full["thresh"])
    del full
    gout, (qd, kd, _) = _run(w.entry, q, k, v, tau, w.sink_start, w.sink_tokens)
    exact, total, mn, mx = sa.last_stats()
    gmask, gthr = sa.debug_route(qd, kd, tau, w.sink_start, w.sink_tokens)
    gm = gmask.cpu().numpy()
    skip = check_mask(gm, ref, orc.sink_block_flags(w.N, w.sink_start, w.sink_tokens))
    assert skip.mean() <= 0.01
    assert exact == int(gm.sum()) and total == gm.size
    assert abs((1 - exact / total) - w.target_sparsity) < 0.01
    np.testing.assert_allclose(gthr.cpu().numpy(), ref["thresh"], rtol=1e-5, atol=2e-6)
    # rows of sampled query blocks whose masks differ: the oracle with the GPU's exact sets
    skip &= np.isin(np.arange(Nb), sample)[None, None, :]
    args = (q, k, v, tau, w.sink_start, w.sink_tokens)
    compare_outputs(gout, with_gpu_mask(fn, args, gm, skip, ref["out"]), w.N)


def test_repeated_calls_are_bitwise_identical():
    q, k, v = _to_gpu(*iid_qkv(1, 3000, 4, seed=5))
    a = sa.sol_attn_fwd(q, k, v, 1.0)
    b = sa.sol_attn_fwd(q, k, v, 1.0)
    c = sa.sol_attn2_fwd(q, k, v, 1.0)
    d = sa.sol_attn2_fwd(q, k, v, 1.0)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(c, d)


def test_argument_errors_are_reported_before_launch():
    q, k, v = _to_gpu(*iid_qkv(1, 256, 2, seed=1))
    with pytest.raises(sa.SolAttnError) as e:
        sa.sol_attn_fwd(q, k, v, float("nan"))
    assert e.value.code == -3
    with pytest.raises(sa.SolAttnError) as e:
        sa.sol_attn_fwd(q, k, v, 1.0, sink_start=256, sink_tokens=4)
    assert e.value.code == -4
    with pytest.raises(sa.SolAttnError) as e:
        sa.sol_attn_fwd(q, k, v, 1.0, out=q)
    assert e.value.code == -5
    assert sa.get_device_status() == 0


def test_stream_and_stats_and_timing():
    q, k, v = _to_gpu(*iid_qkv(1, 2048, 2, seed=2))
    s = torch.cuda.Stream()
    sa.set_kernel_timing(True)
    with torch.cuda.stream(s):
        out = sa.sol_attn_fwd(q, k, v, 1.0, stream=s)
    ms = sa.last_kernel_ms()
    sa.set_kernel_timing(False)
    s.synchronize()
    ref = sa.sol_attn_fwd(q, k, v, 1.0)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert ms > 0
    exact, total, mn, mx = sa.last_stats()
    assert total == 2 * 32 * 32 and 0 < exact <= total and 2 <= mn <= mx <= 32
    assert sa.last_launch_count() == 7


def test_unit_timing_records_every_work_unit():
    """Per-CTA timing of the fused kernel: one record per 128-row query tile, each inside the launch
    window, on a valid SM, and the output unchanged by the recording."""
    q, k, v = _to_gpu(*iid_qkv(2, 3000, 3, seed=8))
    ref = sa.sol_attn_fwd(q, k, v, 1.0)
    sa.set_unit_timing(True)
    try:
        out = sa.sol_attn_fwd(q, k, v, 1.0)
        torch.cuda.synchronize()
        ut = sa.last_unit_times()
    finally:
        sa.set_unit_timing(False)
    assert torch.equal(out, ref)
    Nb = (3000 + 63) // 64
    assert ut.shape == (2 * 3 * ((Nb + 1) // 2), 3)
    assert (ut[:, 1] > ut[:, 0]).all() and (ut[:, 0] > 0).all()
    assert (ut[:, 1].max() - ut[:, 0].min()) < 1e9                  # one launch, well under a second
    assert ((ut[:, 2] >= 0) & (ut[:, 2] < torch.cuda.get_device_properties(0).multi_processor_count)).all()


@pytest.mark.parametrize("name", ["tiny", "wan"])
def test_diagonal_threshold_estimator(name):
    """thresh_type="diag" (appendix "Diagonal threshold estimator") against the oracle."""
    w = WORKLOADS[name]
    q, k, v = w.make_inputs("cpu")
    tau = w.resolved_tau()
    ref = orc.sol_attn(q, k, v, tau, w.sink_start, w.sink_tokens, thresh_type="diag")
    full = orc.routing(q, k, tau, w.sink_start, w.sink_tokens, thresh_type="diag")
    ref.update(shat=full["shat"], thresh=full["thresh"])
    qd, kd, vd = _to_gpu(q, k, v)
    out = sa.sol_attn_fwd(qd, kd, vd, tau, w.sink_start, w.sink_tokens, thresh_type="diag")
    torch.cuda.synchronize()
    assert sa.get_device_status() == 0
    gmask, gthr = sa.debug_route(qd, kd, tau, w.sink_start, w.sink_tokens, thresh_type="diag")
    gm = gmask.cpu().numpy()
    skip = check_mask(gm, ref)
    np.testing.assert_allclose(gthr.cpu().numpy(), full["thresh"], rtol=1e-5, atol=2e-6)
    args = (q, k, v, tau, w.sink_start, w.sink_tokens)
    compare_outputs(out.float().cpu().numpy(), with_gpu_mask(orc.sol_attn, args, gm, skip, ref["out"], thresh_type="diag"),
                    w.N)
    exact = orc.routing(q, k, tau, w.sink_start, w.sink_tokens)
    assert not np.array_equal(exact["mask"], full["mask"])   # the estimator changes the routing


@pytest.mark.parametrize("entry", ["sol_attn", "sol_attn2"])
def test_extra_sink_ranges(entry):
    """Several exact key ranges (the main sink plus extra ranges from the options) against the oracle."""
    B, N, H, tau = 1, 3000, 2, 2.0
    extra = [(900, 30), (2100, 200), (2990, 50)]
    q, k, v = iid_qkv(B, N, H, seed=77)
    fn = orc.sol_attn if entry == "sol_attn" else orc.sol_attn2
    ref = fn(q, k, v, tau, 0, 100, extra_sinks=extra)
    full = orc.routing(q, k, tau, 0, 100, extra_sinks=extra)
    ref.update(shat=full["shat"], thresh=full["thresh"])
    qd, kd, vd = _to_gpu(q, k, v)
    gfn = sa.sol_attn_fwd if entry == "sol_attn" else sa.sol_attn2_fwd
    out = gfn(qd, kd, vd, tau, 0, 100, extra_sinks=extra)
    torch.cuda.synchronize()
    assert sa.get_device_status() == 0
    gmask, _ = sa.debug_route(qd, kd, tau, 0, 100, extra_sinks=extra)
    flags = orc.sink_block_flags(N, 0, 100, extra)
    assert flags.sum() >= 7
    gm = gmask.cpu().numpy()
    skip = check_mask(gm, ref, sink_flags=flags)
    compare_outputs(out.float().cpu().numpy(),
                    with_gpu_mask(fn, (q, k, v, tau, 0, 100), gm, skip, ref["out"], extra_sinks=extra), N)


@pytest.mark.parametrize("rows", [(70, 131), (0, 64), (-1, 40), (1500, 10_000)])
def test_dense_rows_companion(rows):
    """sol_attn_dense_rows: the given query rows get dense attention, every other row is untouched."""
    B, N, H = 1, 2000, 2
    q, k, v = iid_qkv(B, N, H, seed=91)
    qd, kd, vd = _to_gpu(q, k, v)
    out = sa.sol_attn_fwd(qd, kd, vd, 1.0, 0, 128)
    before = out.clone()
    sa.sol_attn_dense_rows(qd, kd, vd, out, rows[0], rows[1])
    torch.cuda.synchronize()
    assert sa.get_device_status() == 0
    ref = orc.dense_rows(q, k, v, rows[0], rows[1])
    sel = ~np.isnan(ref[0, :, 0, 0])
    assert sel.any()
    compare_outputs(out.float().cpu().numpy(), ref, N)
    untouched = torch.from_numpy(~sel).to(out.device)
    assert torch.equal(out[0][untouched], before[0][untouched])


@pytest.mark.parametrize("kv_splits", [2, 4, 8])
@pytest.mark.parametrize("case", [("n129", 1, 129, 2, 1.0, -1, 0), ("n1000_b2", 2, 1000, 2, 1.0, -1, 0),
                                  ("n4000_high_tau", 1, 4000, 2, 3.0, -1, 0)], ids=lambda c: c[0])
def test_split_kv(case, kv_splits):
    """kv_splits > 1 (README "Long-sequence tuning"): shares of each query tile's key tiles on separate
    CTAs, merged by the combine kernel; the same oracle result (n129 with 8 splits leaves most shares
    empty)."""
    name, B, N, H, tau, ss, st = case
    q, k, v = _small_inputs(name, B, N, H)
    ref = orc.sol_attn(q, k, v, tau, ss, st)
    qd, kd, vd = _to_gpu(q, k, v)
    out = sa.sol_attn_fwd(qd, kd, vd, tau, ss, st, kv_splits=kv_splits)
    torch.cuda.synchronize()
    assert sa.get_device_status() == 0
    assert sa.last_launch_count() == 8   # routing (6) + fused kernel + combine
    gmask, _ = sa.debug_route(qd, kd, tau, ss, st)
    gm = gmask.cpu().numpy()
    skip = check_mask(gm, ref)
    compare_outputs(out.float().cpu().numpy(), with_gpu_mask(orc.sol_attn, (q, k, v, tau, ss, st), gm, skip, ref["out"]),
                    N)
    one = sa.sol_attn_fwd(qd, kd, vd, tau, ss, st)
    torch.cuda.synchronize()
    assert (out.float() - one.float()).abs().max().item() <= 1.6e-2


@pytest.mark.parametrize("entry", ["sol_attn", "sol_attn2"])
@pytest.mark.parametrize("case", [("n129", 1, 129, 2, 1.0, -1, 0), ("n1000_b2", 2, 1000, 2, 1.0, -1, 0),
                                  ("n1000_interior_sink", 1, 1000, 2, 1.5, 300, 200),
                                  ("n4000_high_tau", 1, 4000, 2, 3.0, -1, 0)], ids=lambda c: c[0])
def test_m_tile_64(case, entry):
    """m_tile = 64 (one query block per work unit, README per-shape tuning): the oracle's result,
    and the default tiling's up to FP32 rounding; odd and even block counts, a ragged last block."""
    name, B, N, H, tau, ss, st = case
    q, k, v = _small_inputs(name, B, N, H)
    fn = getattr(orc, entry)
    ref = fn(q, k, v, tau, ss, st)
    qd, kd, vd = _to_gpu(q, k, v)
    gfn = sa.sol_attn_fwd if entry == "sol_attn" else sa.sol_attn2_fwd
    out = gfn(qd, kd, vd, tau, ss, st, m_tile=64)
    torch.cuda.synchronize()
    assert sa.get_device_status() == 0
    gmask, _ = sa.debug_route(qd, kd, tau, ss, st)
    gm = gmask.cpu().numpy()
    skip = check_mask(gm, ref, orc.sink_block_flags(N, ss, st))
    compare_outputs(out.float().cpu().numpy(), with_gpu_mask(fn, (q, k, v, tau, ss, st), gm, skip, ref["out"]), N)
    default = gfn(qd, kd, vd, tau, ss, st)
    torch.cuda.synchronize()
    assert (out.float() - default.float()).abs().max().item() <= 1.6e-2


@pytest.mark.parametrize("entry", ["sol_attn", "sol_attn2"])
def test_host_buffer_entry_points_match_the_device_call(entry):
    """sol_attn_fwd_host / sol_attn2_fwd_host: pinned host tensors in and out, (b, head-chunk) slices
    pipelined; each slice is an independent call, so the result equals the device call bit for bit
    (B = 2, H = 5 heads in chunks of 2, the last one short)."""
    q, k, v = iid_qkv(2, 1500, 5, seed=19)
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    host_fn = sa.sol_attn_fwd_host if entry == "sol_attn" else sa.sol_attn2_fwd_host
    dev_fn = sa.sol_attn_fwd if entry == "sol_attn" else sa.sol_attn2_fwd
    out = host_fn(qh, kh, vh, 1.0, 0, 64, heads_per_chunk=2)
    ref = dev_fn(*_to_gpu(q, k, v), 1.0, 0, 64)
    torch.cuda.synchronize()
    assert sa.get_device_status() == 0
    assert out.device.type == "cpu" and torch.equal(out, ref.cpu())
    again = host_fn(q, k, v, 1.0, 0, 64)          # pageable buffers, default chunking
    assert torch.equal(again, out)


def test_split_kv_is_sol_attn_only():
    q, k, v = _to_gpu(*iid_qkv(1, 256, 1, seed=3))
    with pytest.raises(sa.SolAttnError):
        sa._fwd("sol_attn2_fwd", q, k, v, 1.0, -1, 0, None, None, "exact", (), 2)


def test_varlen_packed_batch():
    """sol_attn_fwd_varlen: packed sequences of different lengths (one empty), each against the oracle
    on its own tokens, with a per-sequence prefix sink."""
    H, tau = 2, 1.0
    lens = [700, 0, 64, 1300]
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    q, k, v = iid_qkv(1, cu[-1], H, seed=55)
    out = sa.sol_attn_fwd_varlen(*(t[0].cuda() for t in (q, k, v)), cu, tau, 0, 32)
    torch.cuda.synchronize()
    assert sa.get_device_status() == 0
    got = out.float().cpu().numpy()
    for s, n in enumerate(lens):
        if n == 0:
            continue
        sl = slice(cu[s], cu[s + 1])
        qs, ks, vs = q[:, sl], k[:, sl], v[:, sl]
        ref = orc.sol_attn(qs, ks, vs, tau, 0, 32)
        gmask, _ = sa.debug_route(qs.cuda(), ks.cuda(), tau, 0, 32)
        gm = gmask.cpu().numpy()
        skip = check_mask(gm, ref)
        compare_outputs(got[None, sl], with_gpu_mask(orc.sol_attn, (qs, ks, vs, tau, 0, 32), gm, skip, ref["out"]), n)
