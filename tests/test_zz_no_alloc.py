"""The allocation-free entry point (sol_attn_fwd_noalloc) against sol_attn_fwd, through the C ABI.

Callers that cannot allocate device memory during a call (a caller-managed memory pool, a runtime
that reserved the device's memory up front) use sol_attn_fwd_noalloc, whose scratch is a fixed
region inside the library.  This file sorts last so that a run stopping at the first failure has
already run every other test; it passes in a fresh process as well (the first call on the device
does the region's set-up).
"""
import ctypes

import pytest
import torch

from block_sparse_attention_sum_b200 import sol_attn as sa
from block_sparse_attention_sum_b200.inputs import iid_qkv
from block_sparse_attention_sum_b200.workloads import WORKLOADS
from tests.parity import MAX_ABS, REL_L2

pytestmark = pytest.mark.gpu


def _close(a, b):
    d = (a.float() - b.float())
    assert torch.isfinite(a.float()).all()
    assert d.abs().max().item() <= MAX_ABS
    assert (d.norm() / b.float().norm()).item() <= REL_L2


@pytest.mark.parametrize("case", [("tiny", None), ("ragged", (2, 1000, 3, 1.0, -1, 10)), ("wan", None)])
def test_noalloc_matches_pooled_entry_on_two_calls(case):
    name, shape = case
    if shape is None:
        w = WORKLOADS[name]
        q, k, v = (t.cuda() for t in w.make_inputs("cpu"))
        tau, ss, st = w.resolved_tau(), w.sink_start, w.sink_tokens
    else:
        B, N, H, tau, ss, st = shape
        q, k, v = (t.cuda() for t in iid_qkv(B, N, H, seed=3))
    ref = sa.sol_attn_fwd(q, k, v, tau, ss, st)
    lib = sa.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):   # the second call reuses the scratch left by the first
        out = torch.full_like(q, float("nan"))
        rc = lib.sol_attn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), q.shape[0],
                                      q.shape[1], q.shape[2], float(tau), ss, st, stream)
        assert rc == 0, lib.sol_attn_last_error()
        assert lib.sol_attn_noalloc_get_device_status(stream) == 0, lib.sol_attn_last_error()
        _close(out, ref)
        # the same kernels on the same inputs: the result is the pooled entry point's, bit for bit
        # (stale scratch from an earlier call would show here first)
        assert torch.equal(out, ref)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    q = torch.zeros(1, 65536, 32, 128, dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    lib = sa.load_library()
    rc = lib.sol_attn_fwd_noalloc(q.data_ptr(), q.data_ptr(), q.data_ptr(), out.data_ptr(), 1, 65536, 32, 1.0, -1,
                                  0, None)
    assert rc == -2
    assert b"scratch" in lib.sol_attn_last_error()
