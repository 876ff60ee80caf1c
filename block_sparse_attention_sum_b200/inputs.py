"""Seeded synthetic Q/K/V generators shared by the CUDA path's tests, the bench and the oracle.

This module only synthesises data. It holds none of the attention method's arithmetic, so the
oracle and the CUDA path can both consume its tensors without sharing any of the method.

Two families of inputs stand in for the model activations the pages measure on (Wan2.1,
HunyuanVideo and other diffusion transformers, Sol-Attn paper, arXiv 2607.24027, section 4.1):

* ``iid``  -- i.i.d. standard normal values (the tiny operator check).
* ``grf``  -- per (batch, head, channel) a unit-variance Gaussian random field on the latent
  video grid (T, Y, X), correlation exp(-r^2 / (2 L^2)) with correlation length L cells, plus
  ``noise`` times i.i.d. N(0, 1).  The grid is flattened t-major (token = (t*Y + y)*X + x), the
  order in which video latents are fed to the attention layer.

All tensors are returned in BF16 with layout BTHD ([B, N, H, 128]), rounded to nearest even from
the FP32 values.  The same seed gives the same tensor on the same device type; CPU and CUDA
random streams differ, so a test that compares two implementations generates once and hands the
same tensor (or a host copy of it) to both.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

HEAD_DIM = 128


@dataclass(frozen=True)
class GridSpec:
    """Latent video grid (frames, rows, columns); tokens = T * Y * X, flattened t-major."""

    T: int
    Y: int
    X: int

    @property
    def tokens(self) -> int:
        return self.T * self.Y * self.X


def iid_qkv(B: int, N: int, H: int, seed: int = 0, device: str | torch.device = "cpu"):
    """q, k, v drawn in that order from one generator seeded with ``seed`` (N(0,1), then BF16)."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(seed)
    out = []
    for _ in range(3):
        x = torch.randn(B, N, H, HEAD_DIM, generator=gen, device=dev, dtype=torch.float32)
        out.append(x.to(torch.bfloat16))
    return tuple(out)


def _gaussian_transfer(grid: GridSpec, corr_len: float, device) -> tuple[torch.Tensor, float]:
    """Fourier-domain Gaussian filter on the periodic grid and the variance it gives unit white noise.

    Filtering white noise with a Gaussian kernel of std s gives a field whose autocorrelation is a
    Gaussian of std s*sqrt(2); s = L/sqrt(2) therefore yields correlation exp(-r^2/(2 L^2)).
    The variance of the filtered field is the mean of |H(f)|^2 over the full spectrum (Parseval).
    """
    s = corr_len / math.sqrt(2.0)
    ft = torch.fft.fftfreq(grid.T, device=device, dtype=torch.float64)
    fy = torch.fft.fftfreq(grid.Y, device=device, dtype=torch.float64)
    fx_full = torch.fft.fftfreq(grid.X, device=device, dtype=torch.float64)
    fx = torch.fft.rfftfreq(grid.X, device=device, dtype=torch.float64)

    def transfer(fx_axis):
        f2 = ft[:, None, None] ** 2 + fy[None, :, None] ** 2 + fx_axis[None, None, :] ** 2
        return torch.exp(-2.0 * math.pi**2 * s * s * f2)

    var = float((transfer(fx_full) ** 2).mean())
    return transfer(fx).to(torch.float32), var


def grf_tensor(B: int, H: int, grid: GridSpec, seed: int, corr_len: float = 4.0, noise: float = 0.5,
               device: str | torch.device = "cpu", chunk: int = 256) -> torch.Tensor:
    """One BF16 [B, N, H, 128] tensor: unit-variance GRF per (b, h, channel) + noise * N(0, 1).

    Fields are drawn in (b, h, channel) order from one generator seeded with ``seed``: for each
    chunk of fields, first the white noise that is filtered, then the additive i.i.d. noise.
    """
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(seed)
    Hf, var = _gaussian_transfer(grid, corr_len, dev)
    norm = 1.0 / math.sqrt(var)
    n_fields = B * H * HEAD_DIM
    N = grid.tokens
    out = torch.empty(B, N, H, HEAD_DIM, dtype=torch.bfloat16, device=dev)
    out_fields = out.view(B, N, H * HEAD_DIM)
    for f0 in range(0, n_fields, chunk):
        f1 = min(n_fields, f0 + chunk)
        w = torch.randn(f1 - f0, grid.T, grid.Y, grid.X, generator=gen, device=dev, dtype=torch.float32)
        field = torch.fft.irfftn(torch.fft.rfftn(w, dim=(1, 2, 3)) * Hf, s=(grid.T, grid.Y, grid.X), dim=(1, 2, 3))
        field = field * norm
        field = field + noise * torch.randn(field.shape, generator=gen, device=dev, dtype=torch.float32)
        field = field.reshape(f1 - f0, N)
        # field index f -> (b, h*128 + c)
        for b in range(f0 // (H * HEAD_DIM), (f1 - 1) // (H * HEAD_DIM) + 1):
            lo = max(f0, b * H * HEAD_DIM)
            hi = min(f1, (b + 1) * H * HEAD_DIM)
            out_fields[b, :, lo - b * H * HEAD_DIM: hi - b * H * HEAD_DIM] = (
                field[lo - f0: hi - f0].t().to(torch.bfloat16))
    return out


def grf_qkv(B: int, H: int, grid: GridSpec, seed_base: int, corr_len: float = 4.0, noise: float = 0.5,
            device: str | torch.device = "cpu"):
    """q, k, v as independent fields with seeds seed_base + 0, 1, 2."""
    return tuple(grf_tensor(B, H, grid, seed_base + t, corr_len, noise, device) for t in range(3))
