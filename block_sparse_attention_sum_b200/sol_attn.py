"""Python binding of the C ABI in include/sol_attn.h (argument marshalling only).

Every step of the operator runs in the CUDA library ``libsolattn.so`` built in this directory; there
is no fallback.  If the library is missing, every call raises.  PyTorch provides device memory and
streams only.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

HEAD_DIM = 128
BLOCK = 64
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsolattn.so")

# include/sol_attn.h, in declaration order
EXPORTS = [
    "sol_attn_fwd",
    "sol_attn2_fwd",
    "sol_attn_fwd_ex",
    "sol_attn2_fwd_ex",
    "sol_attn_debug_route_ex",
    "sol_attn_last_error",
    "sol_attn_get_device_status",
    "sol_attn_debug_route",
    "sol_attn_last_stats",
    "sol_attn_set_kernel_timing",
    "sol_attn_last_kernel_ms",
    "sol_attn_kernel_ms_sum",
    "sol_attn_set_unit_timing",
    "sol_attn_last_unit_times",
    "sol_attn_last_launch_count",
    "sol_attn_release_workspace",
    "sol_attn_fwd_noalloc",
    "sol_attn_noalloc_get_device_status",
    "sol_attn_fwd_varlen",
    "sol_attn_dense_rows",
    "sol_attn_set_workspace_limit",
    "sol_attn_selftest_wait_timeout",
    "sol_attn_fwd_host",
    "sol_attn2_fwd_host",
    "sol_attn_fwd_fp8",
    "sol_attn2_fwd_fp8",
    "sol_attn_expcast_host",
    "sol_attn_quot448_host",
]

STATUS = {
    0: "SOL_OK", -1: "SOL_ERR_NULL", -2: "SOL_ERR_SHAPE", -3: "SOL_ERR_TAU", -4: "SOL_ERR_SINK",
    -5: "SOL_ERR_ALIGN", -6: "SOL_ERR_ALLOC", -7: "SOL_ERR_LAUNCH", -8: "SOL_ERR_DEVICE", -9: "SOL_ERR_TIMEOUT",
    -10: "SOL_ERR_OPTION",
}

THRESH_TYPES = {"exact": 0, "diag": 1}
PRECISIONS = {"bf16": 0, "fp8": 1}
MAX_EXTRA_SINKS = 4
MAX_KV_SPLITS = 8


class Options(ctypes.Structure):
    """sol_attn_options (include/sol_attn.h)."""

    _fields_ = [("thresh_type", ctypes.c_int), ("n_extra_sinks", ctypes.c_int),
                ("extra_sink_start", ctypes.c_int * MAX_EXTRA_SINKS), ("extra_sink_tokens", ctypes.c_int * MAX_EXTRA_SINKS),
                ("kv_splits", ctypes.c_int), ("precision", ctypes.c_int), ("m_tile", ctypes.c_int),
                ("reserved", ctypes.c_int * 3)]


def _options(thresh_type: str, extra_sinks=(), kv_splits: int = 1, precision: str = "bf16", m_tile: int = 128):
    """extra_sinks: up to MAX_EXTRA_SINKS (start, tokens) token ranges made exact for every query;
    kv_splits: split-KV shares per query tile (1 = off); precision: "bf16" or "fp8" (E4M3 + ExpCast);
    m_tile: query rows per work unit of the fused kernel (128: two query blocks, 64: one)."""
    if thresh_type not in THRESH_TYPES:
        raise ValueError(f"thresh_type must be one of {sorted(THRESH_TYPES)}")
    if precision not in PRECISIONS:
        raise ValueError(f"precision must be one of {sorted(PRECISIONS)}")
    extra_sinks = list(extra_sinks)
    if len(extra_sinks) > MAX_EXTRA_SINKS:
        raise ValueError(f"at most {MAX_EXTRA_SINKS} extra sink ranges")
    o = Options()
    o.thresh_type = THRESH_TYPES[thresh_type]
    o.n_extra_sinks = len(extra_sinks)
    o.kv_splits = int(kv_splits)
    o.precision = PRECISIONS[precision]
    o.m_tile = int(m_tile)
    for e, (start, tokens) in enumerate(extra_sinks):
        o.extra_sink_start[e] = int(start)
        o.extra_sink_tokens[e] = int(tokens)
    return o


class SolAttnError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"{STATUS.get(code, code)}: {message}")
        self.code = code


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"Sol-Attn CUDA library not found at {path}; build it with "
                           "`python -m block_sparse_attention_sum_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fwd_args = [vp, vp, vp, vp, i, i, i, f, i, i, vp]
    lib.sol_attn_fwd.argtypes = fwd_args
    lib.sol_attn_fwd.restype = i
    lib.sol_attn2_fwd.argtypes = fwd_args
    lib.sol_attn2_fwd.restype = i
    op = ctypes.POINTER(Options)
    ex_args = [vp, vp, vp, vp, i, i, i, f, i, i, op, vp]
    lib.sol_attn_fwd_ex.argtypes = ex_args
    lib.sol_attn_fwd_ex.restype = i
    lib.sol_attn2_fwd_ex.argtypes = ex_args
    lib.sol_attn2_fwd_ex.restype = i
    lib.sol_attn_debug_route_ex.argtypes = [vp, vp, i, i, i, f, i, i, op, vp, vp, vp]
    lib.sol_attn_debug_route_ex.restype = i
    lib.sol_attn_last_error.argtypes = []
    lib.sol_attn_last_error.restype = ctypes.c_char_p
    lib.sol_attn_get_device_status.argtypes = [vp]
    lib.sol_attn_get_device_status.restype = i
    lib.sol_attn_debug_route.argtypes = [vp, vp, i, i, i, f, i, i, vp, vp, vp]
    lib.sol_attn_debug_route.restype = i
    ll = ctypes.POINTER(ctypes.c_longlong)
    ip = ctypes.POINTER(ctypes.c_int)
    lib.sol_attn_last_stats.argtypes = [ll, ll, ip, ip]
    lib.sol_attn_last_stats.restype = i
    lib.sol_attn_set_kernel_timing.argtypes = [i]
    lib.sol_attn_set_kernel_timing.restype = i
    lib.sol_attn_last_kernel_ms.argtypes = []
    lib.sol_attn_last_kernel_ms.restype = f
    lib.sol_attn_kernel_ms_sum.argtypes = [i]
    lib.sol_attn_kernel_ms_sum.restype = f
    lib.sol_attn_set_unit_timing.argtypes = [i]
    lib.sol_attn_set_unit_timing.restype = i
    lib.sol_attn_last_unit_times.argtypes = [vp, i, ctypes.POINTER(ctypes.c_int)]
    lib.sol_attn_last_unit_times.restype = i
    lib.sol_attn_last_launch_count.argtypes = []
    lib.sol_attn_last_launch_count.restype = i
    lib.sol_attn_release_workspace.argtypes = []
    lib.sol_attn_release_workspace.restype = None
    lib.sol_attn_fwd_noalloc.argtypes = fwd_args
    lib.sol_attn_fwd_noalloc.restype = i
    lib.sol_attn_noalloc_get_device_status.argtypes = [vp]
    lib.sol_attn_noalloc_get_device_status.restype = i
    lib.sol_attn_dense_rows.argtypes = [vp, vp, vp, vp, i, i, i, i, i, vp]
    lib.sol_attn_dense_rows.restype = i
    lib.sol_attn_fwd_varlen.argtypes = [vp, vp, vp, vp, ctypes.POINTER(ctypes.c_int), i, i, f, i, i, op, vp]
    lib.sol_attn_fwd_varlen.restype = i
    lib.sol_attn_set_workspace_limit.argtypes = [ctypes.c_size_t]
    lib.sol_attn_set_workspace_limit.restype = None
    lib.sol_attn_selftest_wait_timeout.argtypes = [vp]
    lib.sol_attn_selftest_wait_timeout.restype = i
    host_args = [vp, vp, vp, vp, i, i, i, f, i, i, op, i]
    lib.sol_attn_fwd_host.argtypes = host_args
    lib.sol_attn_fwd_host.restype = i
    lib.sol_attn2_fwd_host.argtypes = host_args
    lib.sol_attn2_fwd_host.restype = i
    lib.sol_attn_fwd_fp8.argtypes = ex_args
    lib.sol_attn_fwd_fp8.restype = i
    lib.sol_attn2_fwd_fp8.argtypes = ex_args
    lib.sol_attn2_fwd_fp8.restype = i
    lib.sol_attn_expcast_host.argtypes = [ctypes.POINTER(ctypes.c_float), i, f, f, ctypes.POINTER(ctypes.c_uint)]
    lib.sol_attn_expcast_host.restype = i
    lib.sol_attn_quot448_host.argtypes = [ctypes.POINTER(ctypes.c_float), i, f, ctypes.POINTER(ctypes.c_float)]
    lib.sol_attn_quot448_host.restype = i
    _lib = lib
    return lib


def _check(rc: int):
    if rc != 0:
        msg = load_library().sol_attn_last_error().decode(errors="replace")
        raise SolAttnError(rc, msg)


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_qkv(q, k, v=None, host=False):
    ts = [q, k] if v is None else [q, k, v]
    for t in ts:
        if not isinstance(t, torch.Tensor) or t.is_cuda == host:
            raise ValueError("q, k, v must be " + ("CPU" if host else "CUDA") + " tensors")
        if t.dtype != torch.bfloat16 or t.dim() != 4 or t.shape[-1] != HEAD_DIM or not t.is_contiguous():
            raise ValueError("q, k, v must be contiguous BF16 [B, N, H, 128] (BTHD)")
        if t.shape != q.shape or t.device != q.device:
            raise ValueError("q, k, v must share shape and device")
    return q.shape[0], q.shape[1], q.shape[2]


def _fwd(fn_name, q, k, v, tau, sink_start, sink_tokens, out, stream, thresh_type="exact", extra_sinks=(),
         kv_splits=1, precision="bf16", m_tile=128):
    B, N, H = _check_qkv(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != torch.bfloat16 or not out.is_contiguous() or out.device != q.device:
        raise ValueError("out must be a contiguous BF16 tensor shaped like q")
    lib = load_library()
    args = [q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, N, H, float(tau), int(sink_start),
            int(sink_tokens)]
    with torch.cuda.device(q.device):
        if thresh_type != "exact" or extra_sinks or kv_splits != 1 or precision != "bf16" or m_tile != 128:
            opts = _options(thresh_type, extra_sinks, kv_splits, precision, m_tile)
            rc = getattr(lib, fn_name + "_ex")(*args, ctypes.byref(opts), _stream_handle(stream))
        else:
            rc = getattr(lib, fn_name)(*args, _stream_handle(stream))
    _check(rc)
    return out


def sol_attn_fwd(q, k, v, tau=1.0, sink_start=-1, sink_tokens=0, out=None, stream=None, thresh_type="exact",
                 extra_sinks=(), kv_splits=1, precision="bf16", m_tile=128):
    """Sol-Attn forward through the C ABI; returns ``out`` (BF16 [B, N, H, 128])."""
    return _fwd("sol_attn_fwd", q, k, v, tau, sink_start, sink_tokens, out, stream, thresh_type, extra_sinks,
                kv_splits, precision, m_tile)


def sol_attn2_fwd(q, k, v, tau=1.0, sink_start=-1, sink_tokens=0, out=None, stream=None, thresh_type="exact",
                  extra_sinks=(), precision="bf16", m_tile=128):
    """Sol-Attn2 complementary-tail forward through the C ABI; returns ``out``."""
    return _fwd("sol_attn2_fwd", q, k, v, tau, sink_start, sink_tokens, out, stream, thresh_type, extra_sinks,
                precision=precision, m_tile=m_tile)


def _fwd_host(fn_name, q, k, v, tau, sink_start, sink_tokens, out, thresh_type, extra_sinks, heads_per_chunk):
    B, N, H = _check_qkv(q, k, v, host=True)
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != torch.bfloat16 or not out.is_contiguous() or out.device.type != "cpu":
        raise ValueError("out must be a contiguous BF16 CPU tensor shaped like q")
    opts = _options(thresh_type, extra_sinks)
    lib = load_library()
    rc = getattr(lib, fn_name)(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, N, H, float(tau),
                               int(sink_start), int(sink_tokens), ctypes.byref(opts), int(heads_per_chunk))
    _check(rc)
    return out


def sol_attn_fwd_host(q, k, v, tau=1.0, sink_start=-1, sink_tokens=0, out=None, thresh_type="exact", extra_sinks=(),
                      heads_per_chunk=0):
    """Sol-Attn forward of HOST (CPU) tensors, copies pipelined with the computation on the current
    CUDA device; pin the tensors for overlap.  Returns ``out`` (a CPU tensor)."""
    return _fwd_host("sol_attn_fwd_host", q, k, v, tau, sink_start, sink_tokens, out, thresh_type, extra_sinks,
                     heads_per_chunk)


def sol_attn2_fwd_host(q, k, v, tau=1.0, sink_start=-1, sink_tokens=0, out=None, thresh_type="exact", extra_sinks=(),
                       heads_per_chunk=0):
    """Sol-Attn2 forward of HOST (CPU) tensors (see sol_attn_fwd_host)."""
    return _fwd_host("sol_attn2_fwd_host", q, k, v, tau, sink_start, sink_tokens, out, thresh_type, extra_sinks,
                     heads_per_chunk)


def _fwd_fp8(fn_name, q, k, v, tau, sink_start, sink_tokens, out, stream, thresh_type, extra_sinks):
    B, N, H = _check_qkv(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != torch.bfloat16 or not out.is_contiguous() or out.device != q.device:
        raise ValueError("out must be a contiguous BF16 tensor shaped like q")
    opts = _options(thresh_type, extra_sinks)
    lib = load_library()
    with torch.cuda.device(q.device):
        rc = getattr(lib, fn_name)(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, N, H, float(tau),
                                   int(sink_start), int(sink_tokens), ctypes.byref(opts), _stream_handle(stream))
    _check(rc)
    return out


def sol_attn_fwd_fp8(q, k, v, tau=1.0, sink_start=-1, sink_tokens=0, out=None, stream=None, thresh_type="exact",
                     extra_sinks=()):
    """FP8 (E4M3) + ExpCast Sol-Attn forward: BF16 inputs and output, E4M3 attention products."""
    return _fwd_fp8("sol_attn_fwd_fp8", q, k, v, tau, sink_start, sink_tokens, out, stream, thresh_type, extra_sinks)


def sol_attn2_fwd_fp8(q, k, v, tau=1.0, sink_start=-1, sink_tokens=0, out=None, stream=None, thresh_type="exact",
                      extra_sinks=()):
    """FP8 (E4M3) + ExpCast Sol-Attn2 forward (complementary tail as in the BF16 path)."""
    return _fwd_fp8("sol_attn2_fwd_fp8", q, k, v, tau, sink_start, sink_tokens, out, stream, thresh_type,
                    extra_sinks)


def expcast_host(x, fs: float, pivot: float):
    """The FP8 kernels' ExpCast encoder evaluated on the host: uint8 codes of x * fs - pivot (x a
    sequence of floats, length a multiple of 4), unpacked from the library's 32-bit words."""
    import numpy as np

    xs = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    words = np.zeros(xs.size // 4, dtype=np.uint32)
    lib = load_library()
    rc = lib.sol_attn_expcast_host(xs.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), int(xs.size), float(fs),
                                   float(pivot), words.ctypes.data_as(ctypes.POINTER(ctypes.c_uint)))
    _check(rc)
    return words.view(np.uint8).copy()


def quot448_host(x, m: float):
    """The FP8 quantisers' scaled value x * 448 / m (before the E4M3 rounding) evaluated on the host
    by the kernels' own inline function: float32 array of len(x)."""
    import numpy as np

    xs = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    q = np.empty_like(xs)
    lib = load_library()
    rc = lib.sol_attn_quot448_host(xs.ctypes.data_as(ctypes.POINTER(ctypes.c_float)), int(xs.size), float(m),
                                   q.ctypes.data_as(ctypes.POINTER(ctypes.c_float)))
    _check(rc)
    return q


def sol_attn_fwd_varlen(q, k, v, cu_seqlens, tau=1.0, sink_start=-1, sink_tokens=0, out=None, stream=None,
                        thresh_type="exact", extra_sinks=(), kv_splits=1, precision="bf16"):
    """Packed variable-length batch: q, k, v BF16 [total_tokens, H, 128]; sequence s is the tokens
    cu_seqlens[s] .. cu_seqlens[s + 1] - 1 (a host list of offsets starting at 0)."""
    for t in (q, k, v):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 3 \
                or t.shape[-1] != HEAD_DIM or not t.is_contiguous() or t.shape != q.shape:
            raise ValueError("q, k, v must be contiguous BF16 CUDA tensors [total_tokens, H, 128] of one shape")
    if out is None:
        out = torch.empty_like(q)
    cu = [int(x) for x in cu_seqlens]
    if cu[-1] > q.shape[0]:
        raise ValueError("cu_seqlens exceeds the packed token count")
    arr = (ctypes.c_int * len(cu))(*cu)
    opts = _options(thresh_type, extra_sinks, kv_splits, precision)
    lib = load_library()
    with torch.cuda.device(q.device):
        rc = lib.sol_attn_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), arr, len(cu) - 1,
                                     q.shape[1], float(tau), int(sink_start), int(sink_tokens), ctypes.byref(opts),
                                     _stream_handle(stream))
    _check(rc)
    return out


def sol_attn_dense_rows(q, k, v, out, q_start, q_tokens, stream=None):
    """Exact dense attention for query tokens [q_start, q_start + q_tokens) written into ``out``
    (the other rows are left as they are); ``q_start < 0`` selects the suffix."""
    B, N, H = _check_qkv(q, k, v)
    if out.shape != q.shape or out.dtype != torch.bfloat16 or not out.is_contiguous() or out.device != q.device:
        raise ValueError("out must be a contiguous BF16 tensor shaped like q")
    lib = load_library()
    with torch.cuda.device(q.device):
        rc = lib.sol_attn_dense_rows(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, N, H, int(q_start),
                                     int(q_tokens), _stream_handle(stream))
    _check(rc)
    return out


def sol_attn_fwd_noalloc(q, k, v, tau=1.0, sink_start=-1, sink_tokens=0, out=None, stream=None):
    """Allocation-free Sol-Attn forward (library-owned fixed scratch; see include/sol_attn.h).

    ``out`` should be preallocated by a caller that cannot allocate during the call."""
    return _fwd("sol_attn_fwd_noalloc", q, k, v, tau, sink_start, sink_tokens, out, stream)


def sol_attn(q, k, v, tau=1.0, sink_start=None, sink_tokens=0, out=None):
    """README-style entry: ``sink_start=None`` with ``sink_tokens > 0`` selects a suffix sink."""
    return sol_attn_fwd(q, k, v, tau, -1 if sink_start is None else sink_start, sink_tokens, out)


def sol_attn2(q, k, v, tau=1.0, sink_start=None, sink_tokens=0, out=None):
    return sol_attn2_fwd(q, k, v, tau, -1 if sink_start is None else sink_start, sink_tokens, out)


def debug_route(q, k, tau=1.0, sink_start=-1, sink_tokens=0, stream=None, thresh_type="exact", extra_sinks=()):
    """Exact-block mask (uint8 [B, H, Nb, Nb]) and thresholds (float32 [B, H, Nb]) from the GPU router."""
    B, N, H = _check_qkv(q, k)
    Nb = math.ceil(N / BLOCK)
    mask = torch.empty(B, H, Nb, Nb, dtype=torch.uint8, device=q.device)
    thresh = torch.empty(B, H, Nb, dtype=torch.float32, device=q.device)
    lib = load_library()
    with torch.cuda.device(q.device):
        opts = _options(thresh_type, extra_sinks)
        rc = lib.sol_attn_debug_route_ex(q.data_ptr(), k.data_ptr(), B, N, H, float(tau), int(sink_start),
                                         int(sink_tokens), ctypes.byref(opts), mask.data_ptr(), thresh.data_ptr(),
                                         _stream_handle(stream))
    _check(rc)
    return mask, thresh


def set_unit_timing(enable: bool) -> None:
    _check(load_library().sol_attn_set_unit_timing(1 if enable else 0))


def last_unit_times():
    """Per-CTA (start ns, end ns, SM id) of the last timed fused launch, as an int64 array [units, 3]."""
    import numpy as np

    lib = load_library()
    n = ctypes.c_int()
    probe = np.zeros(3, dtype=np.uint64)
    _check(lib.sol_attn_last_unit_times(probe.ctypes.data, 0, ctypes.byref(n)))
    buf = np.zeros(3 * n.value, dtype=np.uint64)
    _check(lib.sol_attn_last_unit_times(buf.ctypes.data, n.value, ctypes.byref(n)))
    return buf.reshape(n.value, 3).astype(np.int64)


def last_stats():
    """(exact_pairs, total_pairs, min_row, max_row) of the most recent call on its device."""
    lib = load_library()
    e, t = ctypes.c_longlong(), ctypes.c_longlong()
    mn, mx = ctypes.c_int(), ctypes.c_int()
    _check(lib.sol_attn_last_stats(ctypes.byref(e), ctypes.byref(t), ctypes.byref(mn), ctypes.byref(mx)))
    return e.value, t.value, mn.value, mx.value


def selftest_wait_timeout(stream=None) -> int:
    """Enqueue the bounded-wait self-test (see include/sol_attn.h); returns its launch status."""
    return load_library().sol_attn_selftest_wait_timeout(_stream_handle(stream))


def get_device_status(stream=None) -> int:
    return load_library().sol_attn_get_device_status(_stream_handle(stream))


def noalloc_get_device_status(stream=None) -> int:
    return load_library().sol_attn_noalloc_get_device_status(_stream_handle(stream))


def set_kernel_timing(enable: bool):
    _check(load_library().sol_attn_set_kernel_timing(1 if enable else 0))


def last_kernel_ms() -> float:
    return float(load_library().sol_attn_last_kernel_ms())


def kernel_ms_sum(n: int) -> float:
    """Summed fused-kernel duration (ms) of the last n timed launches."""
    return float(load_library().sol_attn_kernel_ms_sum(int(n)))


def last_launch_count() -> int:
    return int(load_library().sol_attn_last_launch_count())


def set_workspace_limit(nbytes: int):
    """Cap the library's per-device workspace (0 removes the cap); see include/sol_attn.h."""
    load_library().sol_attn_set_workspace_limit(int(nbytes))


def release_workspace():
    load_library().sol_attn_release_workspace()
