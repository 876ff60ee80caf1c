"""GPU parity of the FP8 (E4M3) + ExpCast entry points against the FP8 reference (oracle/fp8_oracle.py).

The kernels follow the reference's arithmetic: the same E4M3 operands (up to FP32 rounding of
x / s), the same ExpCast codes up to an exact binade shift of the pivot (both pivots are integers in
base 2), FP32 accumulation.  They can differ by a code where 8u + 55.65 lies within FP32 rounding of
a rounding boundary (one code is 2^(1/8) in weight), and for weights below 2^-15 of a row's maximum
(the kernels' per-warpgroup online pivot can sit a few binades under the reference's), so the
output tolerance is max-abs 3e-2 and relative l2 5e-3 after the BF16 rounding of the output.

These kernels have not yet run on a GPU.  Until their first supervised run the module is skipped
unless SOL_FP8_GPU=1 is set, so that an unattended GPU suite does not make that first run.
"""
import os
import zlib

import numpy as np
import pytest
import torch

from block_sparse_attention_sum_b200 import sol_attn as sa
from block_sparse_attention_sum_b200.inputs import iid_qkv
from block_sparse_attention_sum_b200.workloads import WORKLOADS
from oracle import fp8_oracle as f8
from oracle import sol_attn_oracle as orc
from tests.parity import check_mask, compare_outputs

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(os.environ.get("SOL_FP8_GPU") != "1",
                                 reason="FP8 kernels not yet run on a GPU: first run is a supervised call")]

FP8_MAX_ABS = 3e-2
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
    skip = check_mask(gmask.cpu().numpy(), ref, orc.sink_block_flags(N, ss, st))
    compare_outputs(gout, ref["out"], N, skip_rows=skip, max_abs_tol=FP8_MAX_ABS, rel_l2_tol=FP8_REL_L2)


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
    skip = check_mask(gmask.cpu().numpy(), ref, orc.sink_block_flags(w.N, w.sink_start, w.sink_tokens))
    assert skip.mean() <= 0.01
    compare_outputs(gout, ref["out"], w.N, skip_rows=skip, max_abs_tol=FP8_MAX_ABS, rel_l2_tol=FP8_REL_L2)


def test_fp8_is_close_to_bf16_and_deterministic():
    q, k, v = (t.cuda() for t in iid_qkv(1, 3000, 4, seed=21))
    a = sa.sol_attn_fwd_fp8(q, k, v, 1.0)
    b = sa.sol_attn_fwd_fp8(q, k, v, 1.0)
    c = sa.sol_attn_fwd(q, k, v, 1.0)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    rel = float((a.float() - c.float()).norm() / c.float().norm())
    assert 0.005 < rel < 0.1, rel
