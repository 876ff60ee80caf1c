"""Device-side failure path on the GPU, without a fault: a bounded wait that can never be satisfied
runs out, the timeout reaches the host through the status word, and the library keeps working."""
import numpy as np
import pytest
import torch

from block_sparse_attention_sum_b200 import sol_attn as sa
from block_sparse_attention_sum_b200.inputs import iid_qkv
from oracle import sol_attn_oracle as orc
from tests.parity import check_mask, compare_outputs, with_gpu_mask

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_is_reported():
    torch.cuda.synchronize()
    assert sa.get_device_status() == 0
    assert sa.selftest_wait_timeout() == 0
    assert sa.get_device_status() == -9          # SOL_ERR_TIMEOUT, read and cleared
    assert b"bounded wait" in sa.load_library().sol_attn_last_error()
    assert sa.get_device_status() == 0
    # the context is intact: a forward call right after still matches the oracle
    q, k, v = iid_qkv(1, 700, 2, seed=12)
    out = sa.sol_attn_fwd(*(t.cuda() for t in (q, k, v)), 1.0)
    torch.cuda.synchronize()
    assert sa.get_device_status() == 0
    ref = orc.sol_attn(q, k, v, 1.0)
    mask, _ = sa.debug_route(q.cuda(), k.cuda(), 1.0)
    gm = mask.cpu().numpy()
    skip = check_mask(gm, ref)
    compare_outputs(out.float().cpu().numpy(), with_gpu_mask(orc.sol_attn, (q, k, v, 1.0), gm, skip, ref["out"]), 700)
