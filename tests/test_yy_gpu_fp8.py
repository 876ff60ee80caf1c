"""GPU parity of the FP8 (E4M3) + ExpCast entry points against the FP8 reference (oracle/fp8_oracle.py).

The kernels follow the reference's arithmetic: the same E4M3 operands (the quantiser keeps exact
midpoints exact), the same ExpCast codes up to an exact binade shift of the pivot (both pivots are
integers in base 2), the denominators as sums of the decoded weights; an FP32 model of the kernels
matches the reference to FP32 rounding on the CPU (tests/test_fp8_algorithm_model.py).  A code can
still differ where a score lies within FP32 rounding of a code boundary (a handful per 10^5
scores), so every case uses the BF16 path's tolerances (max-abs 2e-2, relative l2 5e-3).  The
exact-products case (sparse +-1 Q and K: every product and partial sum exact in any accumulator,
every code line 2.9e-2 or more from a rounding boundary) leaves no room even for that.

First B200 run (n300, one head, both entry points, bounds-checked library): device status 0,
1.08e-2 relative l2 from this reference and 5.4e-2 from the BF16 path, matching the FP32 model of
the kernels (with the quantiser's former order x / (max / 448), which rounds exact E4M3 midpoints
the wrong way) to four digits for both entry points; the quantiser is fixed.  The module sorts
after the parity, debug, failure and rescale GPU tests, so a run that stops at its first failure
has run those.
"""
import zlib

import numpy as np
import pytest
import torch

from block_sparse_attention_sum_b200 import sol_attn as sa
from block_sparse_attention_sum_b200.inputs import iid_qkv
from block_sparse_attention_sum_b200.workloads import WORKLOADS
from oracle import fp8_oracle as f8
from oracle import sol_attn_oracle as orc
from tests.parity import check_mask, compare_outputs, model_rows_with_agreeing_masks, with_gpu_mask

pytestmark = pytest.mark.gpu

FP8_MAX_ABS = 2e-2     # the BF16 path's tolerances (module docstring)
FP8_REL_L2 = 5e-3

REF = {"sol_attn": f8.sol_attn_fp8, "sol_attn2": f8.sol_attn2_fp8}
GPU = {"sol_attn": lambda *a, **kw: sa.sol_attn_fwd_fp8(*a, **kw),
       "sol_attn2": lambda *a, **kw: sa.sol_attn2_fwd_fp8(*a, **kw)}


def _run(entry, q, k, v, tau, ss, st):
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out = GPU[entry](qd, kd, vd, tau, ss, st)
    torch.cuda.synchronize()
    assert sa.get_device_status() == 0
    return out.float().cpu().numpy(), (qd, kd, vd)


SMALL = [
    ("n64", 1, 64, 1, 1.0, -1, 0),
    ("n129", 1, 129, 2, 1.0, -1, 0),
    ("n300", 1, 300, 1, 1.0, -1, 0),
    ("n1000_b2_sink", 2, 1000, 2, 1.5, 300, 200),
    ("n4096_low_tau", 1, 4096, 1, -0.5, -1, 0),
]


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
@pytest.mark.parametrize("entry", ["sol_attn", "sol_attn2"])
def test_fp8_small_and_ragged(case, entry):
    name, B, N, H, tau, ss, st = case
    q, k, v = iid_qkv(B, N, H, seed=zlib.crc32(name.encode()) % 1000)
    ref = REF[entry](q, k, v, tau, ss, st)
    gout, (qd, kd, _) = _run(entry, q, k, v, tau, ss, st)
    gmask, _ = sa.debug_route(qd, kd, tau, ss, st)
    full = orc.routing(q, k, tau, ss, st)
    ref.update(shat=full["shat"], thresh=full["thresh"])
    gm = gmask.cpu().numpy()
    skip = check_mask(gm, ref, orc.sink_block_flags(N, ss, st))
    compare_outputs(gout, with_gpu_mask(REF[entry], (q, k, v, tau, ss, st), gm, skip, ref["out"]), N,
                    max_abs_tol=FP8_MAX_ABS, rel_l2_tol=FP8_REL_L2)
    bf = (orc.sol_attn if entry == "sol_attn" else orc.sol_attn2)(q, k, v, tau, ss, st)["out"]
    sel = ~np.isnan(ref["out"])
    assert 3 * np.linalg.norm(gout[sel] - ref["out"][sel]) < np.linalg.norm(gout[sel] - bf[sel])


@pytest.mark.parametrize("name", ["s64k", "sol2_64k"])
def test_fp8_large_workload_sampled(name):
    w = WORKLOADS[name]
    q, k, v = w.make_inputs("cpu")
    tau = w.resolved_tau()
    Nb = orc.num_blocks(w.N)
    sample = sorted(np.random.default_rng(11).choice(Nb, size=8, replace=False).tolist())
    ref = REF[w.entry](q, k, v, tau, w.sink_start, w.sink_tokens, qblocks=sample)
    full = orc.routing(q, k, tau, w.sink_start, w.sink_tokens)
    ref.update(shat=full["shat"], thresh=full["thresh"])
    del full
    gout, (qd, kd, _) = _run(w.entry, q, k, v, tau, w.sink_start, w.sink_tokens)
    gmask, _ = sa.debug_route(qd, kd, tau, w.sink_start, w.sink_tokens)
    gm = gmask.cpu().numpy()
    skip = check_mask(gm, ref, orc.sink_block_flags(w.N, w.sink_start, w.sink_tokens))
    assert skip.mean() <= 0.01
    skip &= np.isin(np.arange(Nb), sample)[None, None, :]
    args = (q, k, v, tau, w.sink_start, w.sink_tokens)
    compare_outputs(gout, with_gpu_mask(REF[w.entry], args, gm, skip, ref["out"]), w.N,
                    max_abs_tol=FP8_MAX_ABS, rel_l2_tol=FP8_REL_L2)


def _sparse_pm1(B, N, H, nnz, seed):
    g = np.random.default_rng(seed)
    x = np.zeros((B, N, H, 128), np.float32)
    for idx in np.ndindex(B, N, H):
        x[idx][g.choice(128, nnz, replace=False)] = g.choice([-1.0, 1.0], nnz)
    return torch.tensor(x).to(torch.bfloat16)


@pytest.mark.parametrize("entry,tau", [("sol_attn2", 1.0), ("sol_attn", -10.0)], ids=["sol_attn2", "sol_attn_dense"])
def test_fp8_exact_products_match_within_bf16_tolerances(entry, tau):
    # tau = -10 makes every block exact, so Sol-Attn has no surrogate tile (whose compressed keys
    # are not exact products)
    N, H = 300, 2
    q, k = _sparse_pm1(1, N, H, 16, 1), _sparse_pm1(1, N, H, 16, 101)
    v = iid_qkv(1, N, H, seed=5)[2]
    ref = REF[entry](q, k, v, tau)
    gout, (qd, kd, _) = _run(entry, q, k, v, tau, -1, 0)
    gmask, _ = sa.debug_route(qd, kd, tau)
    full = orc.routing(q, k, tau)
    ref.update(shat=full["shat"], thresh=full["thresh"])
    gm = gmask.cpu().numpy()
    skip = check_mask(gm, ref)
    if entry == "sol_attn":
        assert gm.all()
    compare_outputs(gout, with_gpu_mask(REF[entry], (q, k, v, tau), gm, skip, ref["out"]), N)


def test_fp8_zero_queries_average_the_values():
    # q = 0: every exact score is 0, every weight an exact power of two (reference pins); V constant
    # over each block and on the E4M3 grid of its head scale
    N, H = 512, 2
    g = np.random.default_rng(3)
    q = torch.zeros(1, N, H, 128, dtype=torch.bfloat16)
    k = torch.tensor(g.standard_normal((1, N, H, 128)), dtype=torch.bfloat16)
    vb = g.choice([-1.0, -0.5, 0.0, 0.5, 1.0], size=(1, N // 64, H, 128))
    vb[0, 0, :, 0] = 1.0
    v = torch.tensor(np.repeat(vb, 64, axis=1), dtype=torch.bfloat16)
    expect = v[0].double().mean(dim=0).numpy()
    for entry in ("sol_attn", "sol_attn2"):
        gout, _ = _run(entry, q, k, v, 1.0, -1, 0)
        np.testing.assert_allclose(gout[0], np.broadcast_to(expect, (N, H, 128)), rtol=0, atol=4e-3)


def test_fp8_is_close_to_bf16_and_deterministic():
    q, k, v = (t.cuda() for t in iid_qkv(1, 3000, 4, seed=21))
    a = sa.sol_attn_fwd_fp8(q, k, v, 1.0)
    b = sa.sol_attn_fwd_fp8(q, k, v, 1.0)
    c = sa.sol_attn_fwd(q, k, v, 1.0)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    rel = float((a.float() - c.float()).norm() / c.float().norm())
    assert 0.005 < rel < 0.1, rel


def test_fp8_precision_option_and_varlen_match_the_fp8_entry_points():
    q, k, v = (t.cuda() for t in iid_qkv(1, 1000, 2, seed=23))
    a = sa.sol_attn_fwd_fp8(q, k, v, 1.0)
    b = sa.sol_attn_fwd(q, k, v, 1.0, precision="fp8")
    c = sa.sol_attn2_fwd_fp8(q, k, v, 1.0)
    d = sa.sol_attn2_fwd(q, k, v, 1.0, precision="fp8")
    cu = [0, 300, 300, 1000]
    pv = sa.sol_attn_fwd_varlen(q[0], k[0], v[0], cu, 1.0, precision="fp8")
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(c, d)
    for s0, s1 in zip(cu[:-1], cu[1:]):
        if s1 > s0:
            one = sa.sol_attn_fwd_fp8(q[:, s0:s1].contiguous(), k[:, s0:s1].contiguous(), v[:, s0:s1].contiguous(), 1.0)
            assert torch.equal(pv[s0:s1], one[0])


@pytest.mark.parametrize("entry", ["sol_attn", "sol_attn2"])
@pytest.mark.parametrize("N,tau,seed,ss,st", [(300, 1.0, 3, -1, 0), (1000, 1.5, 6, 300, 200)], ids=["n300", "n1000_sink"])
def test_fp8_kernel_matches_its_fp32_model(entry, N, tau, seed, ss, st):
    # the FP32 model (tests/test_fp8_algorithm_model.py) follows the kernels' arithmetic step by
    # step, the Sol-Attn2 tail kernel's BF16 operands included (bf16_tail); only the order of the
    # FP32 sums differs, so both round the same values to BF16 except where a score sits within
    # FP32 rounding of a code boundary (a handful of codes per 10^5 scores flip, each moving one
    # key's weight by 2^(1/8)).  Relative l2 1e-3 is below the BF16 rounding floor against the FP64
    # reference (1.65e-3); a systematic slip gives 1e-2.  (With the FP64 tail instead, the model
    # sits 1.372e-3 relative l2 and 1.95e-3 max-abs from itself with the BF16 tail at n300, which is
    # what the GPU showed against it: the tail's BF16 operands, not the FP8 kernel.)
    from tests.test_fp8_algorithm_model import _model_head

    q, k, v = iid_qkv(1, N, 1, seed=seed)
    gout, (qd, kd, _) = _run(entry, q, k, v, tau, ss, st)
    model = _model_head(*(orc.head_slice(t, 0, 0) for t in (q, k, v)), tau, entry == "sol_attn2", ss, st,
                        bf16_tail=True)
    model = torch.tensor(model).to(torch.bfloat16).float().numpy()
    rows = model_rows_with_agreeing_masks(qd, kd, q, k, tau, ss, st)
    d = gout[0, rows, 0] - model[rows]
    assert np.abs(d).max() <= 2e-2 and np.linalg.norm(d) / np.linalg.norm(model[rows]) <= 1e-3

