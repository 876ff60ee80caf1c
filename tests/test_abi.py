"""The C ABI library loads, exports every function the header declares, and rejects bad arguments
on the host before touching a device (CPU only)."""
import ctypes
import os
import re

import pytest

from block_sparse_attention_sum_b200 import sol_attn as sa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sol_attn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(sol_attn\w*)\s*\(", text, flags=re.M)


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_sum_b200.build import build

    build()
    return sa.load_library()


def test_header_and_binding_agree():
    names = declared_functions()
    assert names == sa.EXPORTS


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def _fwd(lib, q=16, k=16, v=16, out=1 << 40, B=1, N=128, H=2, tau=1.0, ss=-1, st=0):
    return lib.sol_attn_fwd(q, k, v, out, B, N, H, tau, ss, st, None)


def test_host_validation_codes(lib):
    assert _fwd(lib, q=0) == -1
    assert _fwd(lib, B=0) == -2 and _fwd(lib, N=-5) == -2 and _fwd(lib, H=0) == -2
    assert _fwd(lib, tau=float("inf")) == -3 and _fwd(lib, tau=float("nan")) == -3
    assert _fwd(lib, ss=128, st=4) == -4
    assert _fwd(lib, q=17) == -5                      # misaligned
    assert _fwd(lib, out=16 + 64) == -5               # out overlaps q, k, v
    assert b"16-byte" in lib.sol_attn_last_error() or len(lib.sol_attn_last_error()) > 0
    assert lib.sol_attn2_fwd(0, 16, 16, 1 << 40, 1, 128, 2, 1.0, -1, 0, None) == -1


def test_no_device_is_an_error_not_a_fallback(lib):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    rc = _fwd(lib)
    assert rc == -8, rc


def test_invalid_options_are_rejected_on_the_host(lib):
    opts = sa.Options(7)
    rc = lib.sol_attn_fwd_ex(16, 16, 16, 1 << 40, 1, 128, 2, 1.0, -1, 0, ctypes.byref(opts), None)
    assert rc == -10
    opts = sa.Options(1)
    opts.reserved[2] = 1
    assert lib.sol_attn2_fwd_ex(16, 16, 16, 1 << 40, 1, 128, 2, 1.0, -1, 0, ctypes.byref(opts), None) == -10
    opts = sa._options("exact", m_tile=96)           # m_tile is 0, 64 or 128
    assert lib.sol_attn_fwd_ex(16, 16, 16, 1 << 40, 1, 128, 2, 1.0, -1, 0, ctypes.byref(opts), None) == -10
    assert b"m_tile" in lib.sol_attn_last_error()
    opts = sa._options("exact", precision="fp8", m_tile=64)   # one-block units: BF16 path only
    assert lib.sol_attn_fwd_ex(16, 16, 16, 1 << 40, 1, 128, 2, 1.0, -1, 0, ctypes.byref(opts), None) == -10
    opts = sa._options("exact", m_tile=64)
    assert lib.sol_attn_fwd_fp8(16, 16, 16, 1 << 40, 1, 128, 2, 1.0, -1, 0, ctypes.byref(opts), None) == -10
    opts = sa._options("exact", [(10, 0)])          # an extra sink needs tokens > 0
    assert lib.sol_attn_fwd_ex(16, 16, 16, 1 << 40, 1, 128, 2, 1.0, -1, 0, ctypes.byref(opts), None) == -10
    opts = sa._options("exact", [(128, 4)])         # start must be < N
    assert lib.sol_attn_fwd_ex(16, 16, 16, 1 << 40, 1, 128, 2, 1.0, -1, 0, ctypes.byref(opts), None) == -10
    opts = sa.Options()
    opts.n_extra_sinks = 5                          # more than SOL_MAX_EXTRA_SINKS
    assert lib.sol_attn_fwd_ex(16, 16, 16, 1 << 40, 1, 128, 2, 1.0, -1, 0, ctypes.byref(opts), None) == -10
    opts = sa.Options()
    opts.extra_sink_tokens[2] = 3                   # an unused slot must stay zero
    assert lib.sol_attn_fwd_ex(16, 16, 16, 1 << 40, 1, 128, 2, 1.0, -1, 0, ctypes.byref(opts), None) == -10
    with pytest.raises(ValueError):
        sa._options("exact", [(0, 1)] * 5)
    opts = sa._options("exact", kv_splits=9)        # more than SOL_MAX_KV_SPLITS
    assert lib.sol_attn_fwd_ex(16, 16, 16, 1 << 40, 1, 128, 2, 1.0, -1, 0, ctypes.byref(opts), None) == -10
    opts = sa._options("exact", kv_splits=-1)
    assert lib.sol_attn_fwd_ex(16, 16, 16, 1 << 40, 1, 128, 2, 1.0, -1, 0, ctypes.byref(opts), None) == -10
    opts = sa.Options()
    opts.precision = 7                              # unknown precision
    assert lib.sol_attn_fwd_ex(16, 16, 16, 1 << 40, 1, 128, 2, 1.0, -1, 0, ctypes.byref(opts), None) == -10
    opts = sa._options("exact", kv_splits=2, precision="fp8")   # no split-KV on the FP8 path
    assert lib.sol_attn_fwd_ex(16, 16, 16, 1 << 40, 1, 128, 2, 1.0, -1, 0, ctypes.byref(opts), None) == -10
    with pytest.raises(ValueError):
        sa._options("exact", precision="fp16")


def test_options_struct_matches_the_header():
    text = open(HEADER).read()
    assert "#define SOL_MAX_EXTRA_SINKS 4" in text and sa.MAX_EXTRA_SINKS == 4
    assert "#define SOL_MAX_KV_SPLITS 8" in text and sa.MAX_KV_SPLITS == 8
    assert ctypes.sizeof(sa.Options) == 16 * 4
    assert "SOL_PRECISION_BF16 = 0" in text and "SOL_PRECISION_FP8 = 1" in text and sa.PRECISIONS == {"bf16": 0, "fp8": 1}
    assert sa.Options.precision.offset == 11 * 4 and sa.Options.m_tile.offset == 12 * 4
    assert sa.Options.reserved.offset == 13 * 4 and "int m_tile;\n  int reserved[3];" in text


def test_dense_rows_host_validation(lib):
    rows = lambda **kw: lib.sol_attn_dense_rows(kw.get("q", 16), 16, 16, kw.get("out", 1 << 40), 1, kw.get("N", 128), 2,
                                                kw.get("qs", 0), kw.get("qt", 10), None)
    assert rows(q=0) == -1
    assert rows(N=0) == -2
    assert rows(qs=128) == -4          # q_start >= N
    assert rows(q=17) == -5
    assert rows(qt=0) == 0             # no rows: nothing to do, no device needed


def test_varlen_host_validation(lib):
    import ctypes as C
    arr = lambda xs: (C.c_int * len(xs))(*xs)
    opts = sa.Options()
    call = lambda cu, n, ss=-1, st=0: lib.sol_attn_fwd_varlen(16, 16, 16, 1 << 40, cu, n, 2, 1.0, ss, st, C.byref(opts), None)
    assert call(None, 1) == -1
    assert call(arr([0, 10]), 0) == -2
    assert call(arr([1, 10]), 1) == -2           # must start at 0
    assert call(arr([0, 10, 5]), 2) == -2        # non-decreasing
    assert call(arr([0, 100, 150]), 2, ss=60, st=4) == -4   # the sink start lies beyond sequence 1
    assert call(arr([0, 0, 0]), 2) == 0          # only empty sequences: nothing to do
