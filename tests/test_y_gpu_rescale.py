"""GPU: rows whose running maximum jumps mid-row, so that the fused kernels' lazy rescaling runs.

Keys of the first half of the sequence are scaled by 0.25 and of the second half by 2, so a row's
maximum grows by about 9 binades after its early tiles: the BF16 kernel's reference maximum moves
(it moves only past 8 binades: in 567 of the 2048 row halves here) and the FP8 kernel's integer
pivot moves (about 4300 times), and O (and the FP8 row sums) are rescaled.  Random inputs almost
never do this.  (A scale of 3 moves nearly every row but makes attention so peaked that outputs
reach 3.4, where BF16 rounding alone uses 40 % of the max-abs tolerance.)

* BF16: rescaling by exact powers of two changes nothing but FP32 rounding, so the kernel must match
  the FP64 reference within the usual tolerances.
* FP8: the pivot is online, as in the pages' description of ExpCast, so weights coded before the
  pivot moved keep codes the final pivot would clip (they sit ~14 binades below the row maximum);
  the reference codes every weight against the final pivot (reading R19) and drops them, which on
  such rows moves the result by several 1e-3 relative l2.  The kernels are therefore compared with their FP32 model,
  which follows the same online pivots (tests/test_fp8_algorithm_model.py).
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_sum_b200 import sol_attn as sa
from block_sparse_attention_sum_b200.inputs import iid_qkv
from oracle import sol_attn_oracle as orc
from tests.parity import check_mask, compare_outputs, model_rows_with_agreeing_masks, with_gpu_mask

pytestmark = pytest.mark.gpu

N = 1024


def _inputs():
    q, k, v = iid_qkv(1, N, 1, seed=31)
    k = k.float()
    k[:, : N // 2] *= 0.25
    k[:, N // 2:] *= 2.0
    return q, k.to(torch.bfloat16), v


@pytest.mark.parametrize("tau", [-10.0, 1.0], ids=["dense", "tau1"])
@pytest.mark.parametrize("entry", ["sol_attn", "sol_attn2"])
def test_bf16_running_max_jump_matches_the_reference(entry, tau):
    q, k, v = _inputs()
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out = (sa.sol_attn_fwd if entry == "sol_attn" else sa.sol_attn2_fwd)(qd, kd, vd, tau)
    torch.cuda.synchronize()
    assert sa.get_device_status() == 0
    ref = getattr(orc, entry)(q, k, v, tau)
    full = orc.routing(q, k, tau)
    ref.update(shat=full["shat"], thresh=full["thresh"])
    gmask, _ = sa.debug_route(qd, kd, tau)
    gm = gmask.cpu().numpy()
    skip = check_mask(gm, ref)
    compare_outputs(out.float().cpu().numpy(), with_gpu_mask(getattr(orc, entry), (q, k, v, tau), gm, skip, ref["out"]), N)


@pytest.mark.parametrize("tau", [-10.0, 1.0], ids=["dense", "tau1"])
@pytest.mark.parametrize("entry", ["sol_attn", "sol_attn2"])
def test_fp8_pivot_jump_matches_the_fp32_model(entry, tau):
    from tests.test_fp8_algorithm_model import _model_head

    q, k, v = _inputs()
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    out = (sa.sol_attn_fwd_fp8 if entry == "sol_attn" else sa.sol_attn2_fwd_fp8)(qd, kd, vd, tau)
    torch.cuda.synchronize()
    assert sa.get_device_status() == 0
    model = _model_head(*(orc.head_slice(t, 0, 0) for t in (q, k, v)), tau, entry == "sol_attn2", bf16_tail=True)
    model = torch.tensor(model).to(torch.bfloat16).float().numpy()
    rows = model_rows_with_agreeing_masks(qd, kd, q, k, tau)
    d = out.float().cpu().numpy()[0, rows, 0] - model[rows]
    assert np.abs(d).max() <= 2e-2 and np.linalg.norm(d) / np.linalg.norm(model[rows]) <= 1e-3
