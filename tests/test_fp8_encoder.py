"""The FP8 kernels' ExpCast encoder (the inline function their softmax runs, evaluated on the host
through sol_attn_expcast_host) against the reference's ExpCast codes; the quantisers' scaled value
x * 448 / m (through sol_attn_quot448_host) against the IEEE division it replaces; and the FP8 entry
points' host-side argument checks (CPU only).

Sol-Attn2 draft, section "FP8 quantization and ExpCast": c(u) = clip_[0,120](RNE(8u + 55.65)) of the
base-2 score u relative to the pivot; codes E4M3(X / s) with s = max |X| / 448."""
import numpy as np
import pytest

from block_sparse_attention_sum_b200 import sol_attn as sa
from oracle import fp8_oracle as f8


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_sum_b200.build import build

    build()
    return sa.load_library()


def _reference_codes(x32, fs, pivot):
    u = x32.astype(np.float64) * np.float64(np.float32(fs)) - pivot
    return f8.expcast_code(u), 8.0 * u + f8.EXPCAST_OFFSET


@pytest.mark.parametrize("seed", range(4))
def test_encoder_matches_the_reference_codes(lib, seed):
    g = np.random.default_rng(seed)
    fs = float(np.float32(g.uniform(0.01, 0.2)))
    pivot = float(g.integers(-40, 40))
    # scores whose u spans the whole code range and below it (u <= 8: the kernels' pivot invariant)
    u = g.uniform(-12.0, 8.0, 40000)
    x = ((u + pivot) / fs).astype(np.float32)
    x = x[(x.astype(np.float64) * fs - pivot) <= 8.0]
    x = x[: len(x) // 4 * 4]
    got = sa.expcast_host(x, fs, pivot).astype(np.int64)
    ref, line = _reference_codes(x, fs, pivot)
    # a code may differ only where 8u + 55.65 sits within FP32 rounding of a rounding boundary
    near_tie = np.abs(line - np.floor(line) - 0.5) < 1e-3
    assert (got[~near_tie] == ref[~near_tie]).all()
    assert (np.abs(got - ref) <= 1).all()
    assert near_tie.mean() < 0.01


def test_encoder_byte_order_masking_and_integer_shifts(lib):
    fs = 0.125
    # u = 0, 1, 2, 3 with pivot 0: codes 56, 64, 72, 80 (2^0 .. 2^3), first in the low byte
    x = np.array([0.0, 8.0, 16.0, 24.0, -np.inf, -np.inf, 0.0, -1e30], dtype=np.float32)
    codes = sa.expcast_host(x, fs, 0.0)
    assert list(codes) == [56, 64, 72, 80, 0, 0, 56, 0]
    assert f8.e4m3_decode(codes[:4]).tolist() == [1.0, 2.0, 4.0, 8.0]
    # an integer change of the pivot moves every normal code by exactly 8 (one binade)
    g = np.random.default_rng(9)
    xs = (g.uniform(-4.0, 6.0, 4096) / fs).astype(np.float32)
    a = sa.expcast_host(xs, fs, 0.0).astype(np.int64)
    b = sa.expcast_host(xs, fs, 1.0).astype(np.int64)
    normal = b >= 8
    assert (a[normal] - b[normal] == 8).all()


def test_encoder_argument_checks(lib):
    with pytest.raises(sa.SolAttnError):
        sa.expcast_host(np.zeros(6, np.float32), 0.1, 0.0)      # n not a multiple of 4
    with pytest.raises(sa.SolAttnError):
        sa.expcast_host(np.zeros(4, np.float32), 0.1, 0.5)      # pivot not an integer
    with pytest.raises(sa.SolAttnError):
        sa.expcast_host(np.zeros(4, np.float32), -1.0, 0.0)     # multiplier not positive


def test_fp8_entry_points_validate_on_the_host(lib):
    import ctypes

    def call(fn, q=16, opts=None, N=128):
        return getattr(lib, fn)(q, 16, 16, 1 << 40, 1, N, 2, 1.0, -1, 0, opts, None)

    for fn in ("sol_attn_fwd_fp8", "sol_attn2_fwd_fp8"):
        assert call(fn, q=0) == -1
        assert call(fn, N=0) == -2
        o = sa.Options()
        o.kv_splits = 2
        assert call(fn, opts=ctypes.byref(o)) == -10                 # no split-KV on the FP8 path
        o = sa.Options()
        o.thresh_type = 7
        assert call(fn, opts=ctypes.byref(o)) == -10


def _bf16_values(lo_bits, hi_bits):
    bits = np.arange(lo_bits, hi_bits, dtype=np.uint32) << 16
    return bits.view(np.float32)


def _assert_same_as_division(x, m):
    import torch

    x = np.asarray(x, dtype=np.float32)
    with np.errstate(over="ignore"):                        # m near the float32 maximum: x * 448 = inf
        ref = (x * np.float32(448.0)) / np.float32(m)      # float32: RN(RN(x * 448) / m)
    got = sa.quot448_host(x, m)
    tiny = np.abs(ref) < 2.0 ** -20                          # E4M3 code +-0 either way (below 2^-10)
    assert np.array_equal(got[~tiny].view(np.uint32), ref[~tiny].view(np.uint32)), m
    assert (np.abs(got[tiny]) < 2.0 ** -20).all() and np.array_equal(np.signbit(got), np.signbit(ref))
    codes = lambda a: torch.from_numpy(a).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes(got), codes(ref))


def test_quantiser_quotient_equals_the_division_for_bf16_blocks(lib):
    # every BF16 x with |x| <= m, both signs, for block maxima m across the exponent range (the
    # reciprocal path covers 2^-100 <= m < 2^101, the division is kept outside it)
    g = np.random.default_rng(3)
    ms = list(_bf16_values(0x0001, 0x7F80)[g.integers(0, 0x7F7F, 160)])
    ms += [2.0 ** -100, 2.0 ** -100 * 0.99, 2.0 ** 100, 2.0 ** 101, 3.875, 1.0, 448.0, 1e-30, 3e38]
    for m in ms:
        m = float(np.float32(m))
        mb = int(np.array([m], dtype=np.float32).view(np.uint32)[0] >> 16)
        x = _bf16_values(0, mb + 1)
        x = x[np.abs(x) <= m]
        _assert_same_as_division(np.concatenate([x, -x]), m)


def test_quantiser_quotient_equals_the_division_for_fp32_values(lib):
    # FP32 inputs (the compressed keys' and values' means) at random magnitudes below m
    g = np.random.default_rng(4)
    for m in np.float32(2.0) ** g.uniform(-60, 60, 200).astype(np.float32) * g.uniform(1, 2, 200).astype(np.float32):
        x = (g.uniform(-1, 1, 5000) * np.float32(2.0) ** g.uniform(-30, 0, 5000)).astype(np.float32) * m
        _assert_same_as_division(x, float(m))


def test_quantiser_quotient_keeps_exact_midpoints_and_signed_zero(lib):
    # 2.90625 * 448 / 3.875 = 336, halfway between the E4M3 values 320 and 352: must stay exact
    q = sa.quot448_host([2.90625, -2.90625, 0.0, -0.0, 3.875], 3.875)
    assert q[0] == 336.0 and q[1] == -336.0 and q[4] == 448.0
    assert q[2] == 0.0 and not np.signbit(q[2]) and q[3] == 0.0 and np.signbit(q[3])


def test_quotient_host_entry_validates_its_arguments(lib):
    import ctypes

    x = (ctypes.c_float * 2)(1.0, 2.0)
    q = (ctypes.c_float * 2)()
    assert lib.sol_attn_quot448_host(None, 2, 1.0, q) == -1                 # SOL_ERR_NULL
    assert lib.sol_attn_quot448_host(x, -1, 1.0, q) == -2                   # SOL_ERR_SHAPE
    for m in (0.0, -1.0, float("inf"), float("nan")):
        assert lib.sol_attn_quot448_host(x, 2, m, q) == -10                 # SOL_ERR_OPTION
    assert lib.sol_attn_quot448_host(x, 0, 1.0, q) == 0
    assert lib.sol_attn_quot448_host(x, 2, 2.0, q) == 0 and list(q) == [224.0, 448.0]
