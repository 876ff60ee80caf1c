"""The seeded generators give the shapes, statistics and determinism the workloads state."""
import math

import torch

from block_sparse_attention_sum_b200.inputs import GridSpec, grf_tensor, iid_qkv
from block_sparse_attention_sum_b200.workloads import WORKLOADS


def test_iid_is_seeded_bf16_bthd():
    a = iid_qkv(1, 256, 2, seed=0)
    b = iid_qkv(1, 256, 2, seed=0)
    assert all(x.dtype == torch.bfloat16 and x.shape == (1, 256, 2, 128) for x in a)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert not torch.equal(a[0], a[1])


def test_grf_variance_and_correlation_length():
    grid = GridSpec(8, 32, 32)
    x = grf_tensor(1, 2, grid, seed=5, noise=0.0).float()          # field only
    assert abs(x.var().item() - 1.0) < 0.05
    f = x[0, :, :, :].reshape(grid.T, grid.Y, grid.X, -1)
    for r in (1, 4):
        c = (f[:, :, r:] * f[:, :, :-r]).mean() / f.var()
        assert abs(c.item() - math.exp(-r * r / 32.0)) < 0.06
    y = grf_tensor(1, 2, grid, seed=5, noise=0.5).float()
    assert abs(y.var().item() - 1.25) < 0.06


def test_workload_shapes():
    w = WORKLOADS["wan"]
    assert w.N == w.grid.tokens == 14040 and w.N % 64 == 24
    assert WORKLOADS["s64k"].N == 65536 and WORKLOADS["s128k"].N == 131072
    assert WORKLOADS["s32k_90"].sink_tokens == 512 and WORKLOADS["s32k_90"].sink_start == 0
