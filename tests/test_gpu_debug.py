"""Debug-build and resource checks on the GPU: the bounds-checked library variant
(-DSOL_ATTN_DEBUG_BOUNDS: every TMA tile coordinate checked against its tensor) runs the small and
ragged shapes without a failed check and with results identical to the release library, and the
workspace cap turns an allocation into SOL_ERR_ALLOC without launching anything."""
import ctypes

import pytest
import torch

from block_sparse_attention_sum_b200 import build as solbuild
from block_sparse_attention_sum_b200 import sol_attn as sa
from block_sparse_attention_sum_b200.inputs import iid_qkv

pytestmark = pytest.mark.gpu

SHAPES = [(1, 64, 1, 1.0, -1, 0), (1, 129, 2, 1.0, -1, 0), (2, 1000, 2, 1.0, 300, 200), (1, 4000, 2, 3.0, -1, 0)]


@pytest.fixture(scope="module")
def debug_lib():
    path = solbuild.build(debug_bounds=True)
    lib = ctypes.CDLL(path)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    for name in ("sol_attn_fwd", "sol_attn2_fwd"):
        getattr(lib, name).argtypes = [vp, vp, vp, vp, i, i, i, f, i, i, vp]
        getattr(lib, name).restype = i
    lib.sol_attn_get_device_status.argtypes = [vp]
    lib.sol_attn_get_device_status.restype = i
    return lib


@pytest.mark.parametrize("entry", ["sol_attn_fwd", "sol_attn2_fwd"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"b{s[0]}n{s[1]}h{s[2]}")
def test_bounds_checked_build_matches_release(debug_lib, entry, shape):
    B, N, H, tau, ss, st = shape
    q, k, v = (t.cuda() for t in iid_qkv(B, N, H, seed=N + B))
    ref = getattr(sa, entry)(q, k, v, tau, ss, st)
    out = torch.full_like(q, float("nan"))
    stream = torch.cuda.current_stream().cuda_stream
    rc = getattr(debug_lib, entry)(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, N, H, tau, ss, st,
                                   stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert debug_lib.sol_attn_get_device_status(stream) == 0   # no bounds check failed, no timeout
    assert torch.equal(out, ref)


def test_workspace_limit_reports_alloc_failure():
    lib = sa.load_library()
    q, k, v = (t.cuda() for t in iid_qkv(1, 8192, 8, seed=4))
    sa.release_workspace()
    lib.sol_attn_set_workspace_limit(1 << 20)
    try:
        with pytest.raises(sa.SolAttnError) as err:
            sa.sol_attn_fwd(q, k, v, 1.0)
        assert err.value.code == -6 and b"limit" in lib.sol_attn_last_error()
    finally:
        lib.sol_attn_set_workspace_limit(0)
    out = sa.sol_attn_fwd(q, k, v, 1.0)
    torch.cuda.synchronize()
    assert sa.get_device_status() == 0 and torch.isfinite(out.float()).all()


def test_debug_route_as_the_first_call_in_a_fresh_process():
    # the routing introspection call must set up everything it uses (the tensor-map encoder among
    # them) when it is the first call of the C ABI a process makes, as __graft_entry__.smoke() does
    import os
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = (
        "import torch\n"
        "from block_sparse_attention_sum_b200 import sol_attn as sa\n"
        "from block_sparse_attention_sum_b200.inputs import iid_qkv\n"
        "q, k, v = (t.cuda() for t in iid_qkv(1, 1024, 2, seed=0))\n"
        "mask, thr = sa.debug_route(q, k, 1.0)\n"
        "out = sa.sol_attn_fwd(q, k, v, 1.0)\n"
        "torch.cuda.synchronize()\n"
        "assert sa.get_device_status() == 0\n"
        "assert bool(mask.any()) and bool(torch.isfinite(out.float()).all())\n"
        "print('ok')\n"
    )
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, (r.returncode, r.stdout[-2000:], r.stderr[-2000:])
    assert r.stdout.strip().endswith("ok")
