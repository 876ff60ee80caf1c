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
    opts.reserved[3] = 1
    assert lib.sol_attn2_fwd_ex(16, 16, 16, 1 << 40, 1, 128, 2, 1.0, -1, 0, ctypes.byref(opts), None) == -10
