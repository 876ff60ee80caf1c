"""Pins for the FP8 + ExpCast reference (CPU only): the E4M3 rounding and decoding against torch's
float8_e4m3fn, ExpCast's exact powers of two and its error bound, the per-block quantiser's
extremes, and a closed form of the whole FP8 forward."""
import math

import numpy as np
import torch

from oracle import fp8_oracle as f8
from oracle import sol_attn_oracle as orc


def test_e4m3_round_matches_torch():
    g = np.random.default_rng(0)
    x = np.concatenate([g.uniform(-448, 448, 4000), g.uniform(-0.05, 0.05, 2000), g.uniform(-1e-3, 1e-3, 500),
                        [0.0, 448.0, -448.0, 1.0625, 1.1875, 2.0 ** -9, 3 * 2.0 ** -10, 0.5 * 2.0 ** -9]])
    ref = torch.tensor(x, dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(f8.e4m3_round(x.astype(np.float32).astype(np.float64)), ref)


def test_e4m3_decode_matches_torch():
    codes = np.arange(0, 127)
    ref = torch.tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(f8.e4m3_decode(codes), ref)
    assert f8.e4m3_decode(126) == 448.0


def test_expcast_powers_of_two_and_error_bound():
    u = np.arange(-6, 9)
    np.testing.assert_array_equal(f8.expcast(u), 2.0 ** u)            # c = 8u + 56 exactly
    assert f8.expcast(-8.0) == 0.0 and f8.expcast_code(-6.96) == 0
    assert f8.expcast_code(20.0) == 120                                # clipped at the top
    assert f8.expcast(20.0) == 256.0                                   # code 120 = 2^8
    t = np.linspace(-6.0, 8.0, 20001)
    rel = np.abs(f8.expcast(t) / 2.0 ** t - 1.0)
    assert rel.max() < 0.075                                           # piecewise-linear mantissa


def test_quantizer_rounds_exact_midpoints_to_even():
    # max 3.8125 (BF16): 448 x / max = -168 exactly for x = -1.4296875, halfway between -160 and -176;
    # ties go to even (-160 = -1.25 * 2^7).  x / (max / 448) in FP64 gives -168.00000000000003.
    x = np.array([-1.4296875, 0.08935546875, 3.8125])
    xq, s = f8.quantize(x)
    np.testing.assert_array_equal(xq / s, [-160.0, 10.0, 448.0])
    assert f8.e4m3_round(-1.4296875 / (3.8125 / 448.0)) == -176.0          # the other order's result
    ref = torch.tensor(x * 448.0 / 3.8125, dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(xq / s, ref)


def test_quantizer_extremes():
    g = np.random.default_rng(1)
    x = g.standard_normal((64, 128)) * 3.0
    xq, s = f8.quantize(x)
    assert math.isclose(s, np.abs(x).max() / 448.0)
    assert np.abs(xq).max() == np.abs(x).max()                         # the extreme maps to +-448 exactly
    big = np.abs(x / s) >= 2.0 ** -6
    assert (np.abs(xq - x)[big] <= 2.0 ** -4 * np.abs(x)[big] + 1e-12).all()
    z, s0 = f8.quantize(np.zeros((10, 128)))
    assert s0 == 1.0 and not z.any()
    blocks = f8.quantize_blocks(np.vstack([x, np.zeros((10, 128))]))  # a partial zero block of 10 rows
    assert not blocks[64:].any() and np.array_equal(blocks[:64], xq)


def test_fp8_forward_with_zero_queries_averages_the_values():
    # q = 0: every exact token has score 0 and every surrogate block log-mass ln 64, so ExpCast gives
    # 2^-6 per token and 1 per block exactly; with V constant over each block and on the E4M3 grid of
    # its head scale (so that the block means are too), the output is the mean of V.
    N, H = 512, 2
    g = np.random.default_rng(3)
    q = np.zeros((1, N, H, 128))
    k = g.standard_normal((1, N, H, 128))
    vb = g.choice([-1.0, -0.5, 0.0, 0.5, 1.0], size=(1, N // 64, H, 128))
    vb[0, 0, :, 0] = 1.0
    v = np.repeat(vb, 64, axis=1)
    out = f8.sol_attn_fp8(q, k, v, tau=1.0)["out"]
    np.testing.assert_allclose(out[0], np.broadcast_to(v[0].mean(axis=0), (N, H, 128)), rtol=0, atol=1e-12)


def test_surrogate_operands_are_quantised_like_keys_and_values():
    # compressed keys: one scale per 64 consecutive block means; compressed values: the head's V scale
    g = np.random.default_rng(6)
    Kbar = g.standard_normal((150, 128))
    Kbar[64:128] *= 100.0                                              # a second group 100x larger
    counts = np.full(150, 64)
    counts[-1] = 17
    Vhat = g.standard_normal((150, 128)) * counts[:, None]
    kbar8, vbar8 = f8.surrogate_operands_fp8(Kbar, Vhat, counts, v_amax=4.48)
    for a, b in ((0, 64), (64, 128), (128, 150)):
        s = np.abs(Kbar[a:b]).max() / 448.0
        np.testing.assert_array_equal(kbar8[a:b], s * f8.e4m3_round(Kbar[a:b] / s))
    vbar = Vhat / counts[:, None]
    np.testing.assert_array_equal(vbar8, (4.48 / 448.0) * f8.e4m3_round(vbar * 448.0 / 4.48))
    assert np.abs(vbar8 - vbar).max() <= 2.0 ** -4 * np.abs(vbar).max()


def test_fp8_forward_reduces_to_the_bf16_path_without_rounding(monkeypatch):
    # with exact exponentials in place of ExpCast and no E4M3 rounding, the FP8 path's algebra
    # (scales, weights, surrogate terms, normaliser) must give the BF16 path's result
    monkeypatch.setattr(f8, "expcast", lambda u: 2.0 ** np.asarray(u))
    monkeypatch.setattr(f8, "e4m3_round", lambda x: np.asarray(x, dtype=np.float64))
    g = np.random.default_rng(4)
    q, k, v = (g.standard_normal((1, 700, 2, 128)) for _ in range(3))
    a = f8.sol_attn_fp8(q, k, v, tau=0.5, sink_start=-1, sink_tokens=30)["out"]
    b = orc.sol_attn(q, k, v, tau=0.5, sink_start=-1, sink_tokens=30)["out"]
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_fp8_forward_error_is_that_of_its_roundings():
    # with the roundings in place the result moves by about the E4M3 / ExpCast resolution (a few
    # percent: 5 % here), not more; a pivot at the row maximum instead of 8 binades below it would
    # drop every weight under 2^-7 of the maximum and double the error
    g = np.random.default_rng(5)
    q, k, v = (g.standard_normal((1, 640, 1, 128)) for _ in range(3))
    a = f8.sol_attn_fp8(q, k, v, tau=1.0)["out"]
    b = orc.sol_attn(q, k, v, tau=1.0)["out"]
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert 0.005 < rel < 0.1, rel


def test_fp8_sol2_reduces_to_the_bf16_sol2_without_rounding(monkeypatch):
    monkeypatch.setattr(f8, "expcast", lambda u: 2.0 ** np.asarray(u))
    monkeypatch.setattr(f8, "e4m3_round", lambda x: np.asarray(x, dtype=np.float64))
    g = np.random.default_rng(7)
    q, k, v = (g.standard_normal((1, 600, 2, 128)) for _ in range(3))
    a = f8.sol_attn2_fp8(q, k, v, tau=0.5, sink_start=0, sink_tokens=64)["out"]
    b = orc.sol_attn2(q, k, v, tau=0.5, sink_start=0, sink_tokens=64)["out"]
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_fp8_sol2_with_zero_queries_averages_the_values():
    # q = 0: exact scores 0 give the ExpCast weight 2^8 (u = 8 against the pivot -8); the tail of an
    # anchor has Z_a = its token count, nu_a = the mean of its values and delta = 0, so with V on the
    # E4M3 grid the output is the mean of V over all tokens.
    N, H = 640, 1
    g = np.random.default_rng(8)
    q = np.zeros((1, N, H, 128))
    k = g.standard_normal((1, N, H, 128))
    v = g.choice([-1.0, -0.5, 0.0, 0.5, 1.0], size=(1, N, H, 128))
    v[0, 0, :, 0] = 1.0
    out = f8.sol_attn2_fp8(q, k, v, tau=1.0)["out"]
    np.testing.assert_allclose(out[0], np.broadcast_to(v[0].mean(axis=0), (N, H, 128)), rtol=0, atol=1e-12)


def test_fp8_sol2_error_is_that_of_its_roundings():
    g = np.random.default_rng(10)
    q, k, v = (g.standard_normal((1, 640, 1, 128)) for _ in range(3))
    a = f8.sol_attn2_fp8(q, k, v, tau=1.0)["out"]
    b = orc.sol_attn2(q, k, v, tau=1.0)["out"]
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert 0.005 < rel < 0.1, rel
