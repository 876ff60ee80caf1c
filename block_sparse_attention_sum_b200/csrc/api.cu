// Host side of the C ABI declared in include/sol_attn.h: argument validation, the per-device
// workspace, TMA descriptors and the launch sequence.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "attn_fwd.cuh"
#include "attn_fwd_fp8.cuh"
#include "fp8.cuh"
#include "common.cuh"
#include "ptx.cuh"
#include "sol_attn.h"

namespace sol {
namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool checked = false;
  bool usable = false;
  void* ws = nullptr;      // workspace
  size_t ws_bytes = 0;
  int* status = nullptr;   // device status word
  unsigned long long* stats = nullptr;
  cudaEvent_t done = nullptr;   // completion of the previous call (cross-stream ordering)
  static constexpr int kRing = 256;
  cudaEvent_t t0[kRing] = {}, t1[kRing] = {};
  int timed_calls = 0;      // timed launches since timing was enabled
  cudaStream_t last_stream = nullptr;
  long long last_total_pairs = 0;
  int last_launches = 0;
  unsigned long long* unit_buf = nullptr;   // per-CTA timing of the fused kernel (when enabled)
  size_t unit_cap = 0;                      // CTAs the buffer holds
  int last_units = 0;                       // CTAs of the last timed fused launch
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

// Host-buffer pipeline of one device: three streams (copies in, compute, copies out), two sets of
// device staging buffers for (b, head-chunk) slices, and the events that order them.
struct HostPipe {
  bool ready = false;
  cudaStream_t in = nullptr, comp = nullptr, out = nullptr;
  cudaEvent_t in_done[2] = {}, comp_done[2] = {}, out_done[2] = {};
  char* buf[2] = {};
  size_t buf_bytes = 0;   // bytes of one set (q, k, v, out slices)
};
std::mutex g_host_mu;     // one host-buffer call at a time (they share the staging buffers)
HostPipe g_pipe[kMaxDevices];
bool g_timing = false;
bool g_unit_timing = false;
int g_last_device = -1;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int get_encode() {
  if (g_encode) return SOL_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr)
    return fail(SOL_ERR_DEVICE, "cuTensorMapEncodeTiled is unavailable");
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return SOL_OK;
}

int device_state(DeviceState** out, int* dev_out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return fail(SOL_ERR_DEVICE, "no current CUDA device");
  DeviceState& d = g_dev[dev];
  if (!d.checked) {
    d.checked = true;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return fail(SOL_ERR_DEVICE, "cudaGetDeviceProperties failed");
    d.usable = prop.major == 10 && prop.minor == 0;
    if (d.usable) {
      if (cudaMalloc(&d.status, sizeof(int)) != cudaSuccess ||
          cudaMalloc(&d.stats, 4 * sizeof(unsigned long long)) != cudaSuccess ||
          cudaMemset(d.status, 0, sizeof(int)) != cudaSuccess ||
          cudaEventCreateWithFlags(&d.done, cudaEventDisableTiming) != cudaSuccess) {
        d.checked = false;
        return fail(SOL_ERR_ALLOC, "device state allocation failed");
      }
    }
  }
  if (!d.usable) return fail(SOL_ERR_DEVICE, "device %d is not an sm_100 (B200-class) GPU", dev);
  *out = &d;
  *dev_out = dev;
  return SOL_OK;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Carves the workspace into the buffers of one call; returns the bytes needed when base == nullptr.
size_t carve(const Shape& s, bool sol2, char* base, Work* w) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off = align_up(off + bytes, 256);
    return p;
  };
  const size_t bh = (size_t)s.BH, nb = (size_t)s.Nb, d = kHeadDim;
  Work t{};
  t.qbar = reinterpret_cast<float*>(take(bh * nb * d * 4));
  t.kbar = reinterpret_cast<float*>(take(bh * nb * d * 4));
  t.kbar_h = reinterpret_cast<__nv_bfloat16*>(take(bh * nb * d * 2));
  t.vbar_h = reinterpret_cast<__nv_bfloat16*>(take(bh * nb * d * 2));
  t.qbar_hi = reinterpret_cast<__nv_bfloat16*>(take(bh * nb * d * 2));
  t.qbar_lo = reinterpret_cast<__nv_bfloat16*>(take(bh * nb * d * 2));
  t.kbar_lo = reinterpret_cast<__nv_bfloat16*>(take(bh * nb * d * 2));
  t.kcov = reinterpret_cast<float*>(take(bh * d * d * 4));
  t.gram_partial = reinterpret_cast<float*>(take(bh * 8 * d * d * 4));
  t.kmean = reinterpret_cast<double*>(take(bh * d * 8));
  t.thresh = reinterpret_cast<float*>(take(bh * nb * 4));
  t.mask = reinterpret_cast<uint32_t*>(take(bh * nb * s.Nw * 4));
  t.rowcount = reinterpret_cast<int*>(take(bh * nb * 4));
  if (sol2) {
    const size_t na = (size_t)s.Na;
    t.qanchor = reinterpret_cast<float*>(take(bh * na * d * 4));
    t.qanchor_h = reinterpret_cast<__nv_bfloat16*>(take(bh * na * d * 2));
    t.qdir = reinterpret_cast<float*>(take(bh * d * 4));
    t.gk_h = reinterpret_cast<__nv_bfloat16*>(take(bh * nb * 2 * d * 2));
    t.gv_h = reinterpret_cast<__nv_bfloat16*>(take(bh * nb * 2 * d * 2));
    t.glog2n = reinterpret_cast<float*>(take(bh * (size_t)tail_groups_padded(s) * 4));
    t.tail_logz = reinterpret_cast<float*>(take(bh * na * 4));
    t.tail_mu = reinterpret_cast<float*>(take(bh * na * d * 4));
    t.tail_nu = reinterpret_cast<float*>(take(bh * na * d * 4));
  }
  if (w) *w = t;
  return off;
}

// The FP8 path's E4M3 operands and scales (after the buffers of carve()); bytes when base == nullptr.
size_t carve_fp8(const Shape& s, char* base, Fp8Work* f) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off = align_up(off + bytes, 256);
    return p;
  };
  const size_t tok = (size_t)s.B * s.N * s.H * kHeadDim, bh = (size_t)s.BH, nbp = (size_t)fp8_rows_padded(s);
  Fp8Work t{};
  t.q8 = reinterpret_cast<uint8_t*>(take(tok));
  t.k8 = reinterpret_cast<uint8_t*>(take(tok));
  t.v8 = reinterpret_cast<uint8_t*>(take(tok));
  t.kbar8 = reinterpret_cast<uint8_t*>(take(bh * nbp * kHeadDim));
  t.vbar8 = reinterpret_cast<uint8_t*>(take(bh * nbp * kHeadDim));
  t.sq = reinterpret_cast<float*>(take(bh * s.Nb * 4));
  t.sk = reinterpret_cast<float*>(take(bh * s.Nb * 4));
  t.skbar = reinterpret_cast<float*>(take(bh * (nbp / 64) * 4));
  t.sv = reinterpret_cast<float*>(take(bh * 4));
  t.vmax = reinterpret_cast<unsigned int*>(take(bh * 4));
  if (f) *f = t;
  return off;
}

// Upper bound on the workspace of one device (0: none); lets callers cap the library's memory and
// lets tests exercise the allocation-failure path without exhausting a GPU.
size_t g_ws_limit = 0;

int ensure_workspace(DeviceState& d, size_t bytes) {
  if (d.ws_bytes >= bytes) return SOL_OK;
  if (g_ws_limit && bytes > g_ws_limit)
    return fail(SOL_ERR_ALLOC, "workspace of %zu bytes exceeds the limit of %zu bytes", bytes, g_ws_limit);
  if (d.ws) {
    cudaDeviceSynchronize();
    cudaFree(d.ws);
    d.ws = nullptr;
    d.ws_bytes = 0;
  }
  size_t grow = align_up(bytes + bytes / 8, 1 << 20);
  if (g_ws_limit && grow > g_ws_limit) grow = bytes;
  if (cudaMalloc(&d.ws, grow) != cudaSuccess) {
    cudaGetLastError();
    return fail(SOL_ERR_ALLOC, "workspace allocation of %zu bytes failed", grow);
  }
  d.ws_bytes = grow;
  return SOL_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

int validate(const void* q, const void* k, const void* v, const void* out, bool need_v_out, int B, int N, int H,
             float tau, int sink_start, int sink_tokens) {
  if (!q || !k || (need_v_out && (!v || !out))) return fail(SOL_ERR_NULL, "q, k, v and out must be non-NULL");
  if (B <= 0 || N <= 0 || H <= 0) return fail(SOL_ERR_SHAPE, "B, N, H must be positive (got %d, %d, %d)", B, N, H);
  const long long elems = (long long)B * N * H * kHeadDim;
  if (elems > (1ll << 40) || (long long)B * H > (1ll << 24) || N > (1 << 30))
    return fail(SOL_ERR_SHAPE, "sizes out of the supported range");
  if (!std::isfinite(tau)) return fail(SOL_ERR_TAU, "tau must be finite");
  if (sink_tokens > 0 && sink_start >= N) return fail(SOL_ERR_SINK, "sink_start (%d) must be < N (%d)", sink_start, N);
  if (!aligned16(q) || !aligned16(k) || (need_v_out && (!aligned16(v) || !aligned16(out))))
    return fail(SOL_ERR_ALIGN, "tensor pointers must be 16-byte aligned");
  if (need_v_out) {
    const size_t bytes = (size_t)elems * 2;
    if (overlaps(out, bytes, q, bytes) || overlaps(out, bytes, k, bytes) || overlaps(out, bytes, v, bytes))
      return fail(SOL_ERR_ALIGN, "out must not overlap q, k or v");
  }
  return SOL_OK;
}

// Adds the key blocks overlapping a sink token range as an inclusive block interval.
void add_sink(int N, int sink_start, int sink_tokens, SinkSet* set) {
  if (sink_tokens <= 0) return;
  long long start = sink_start >= 0 ? sink_start : (long long)N - sink_tokens;
  long long end = start + sink_tokens;
  if (start < 0) start = 0;
  if (end > N) end = N;
  if (end <= start) return;
  set->b0[set->n] = (int)(start / kBlock);
  set->b1[set->n] = (int)((end - 1) / kBlock);
  ++set->n;
}

int encode_bthd(CUtensorMap* m, const void* base, const Shape& s) {
  const cuuint64_t dims[4] = {(cuuint64_t)kHeadDim, (cuuint64_t)s.H, (cuuint64_t)s.N, (cuuint64_t)s.B};
  const cuuint64_t strides[3] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)s.H * kHeadDim * 2,
                                 (cuuint64_t)s.N * s.H * kHeadDim * 2};
  const cuuint32_t box[4] = {64, 1, 64, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SOL_OK : fail(SOL_ERR_LAUNCH, "cuTensorMapEncodeTiled (BTHD) failed: %d", (int)r);
}

// [BH][rows][128] BF16 rows, 64 x 128 x 1 boxes (pooled block means, anchor means, group means)
int encode_rows(CUtensorMap* m, const void* base, int rows, const Shape& s) {
  const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows, (cuuint64_t)s.BH};
  const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)rows * kHeadDim * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SOL_OK : fail(SOL_ERR_LAUNCH, "cuTensorMapEncodeTiled (rows) failed: %d", (int)r);
}

int encode_pooled(CUtensorMap* m, const void* base, const Shape& s) { return encode_rows(m, base, s.Nb, s); }

// E4M3 BTHD bytes: 128 channels x 1 head x 64 tokens x 1 batch boxes (one 128-byte row per token).
int encode_bthd8(CUtensorMap* m, const void* base, const Shape& s) {
  const cuuint64_t dims[4] = {(cuuint64_t)kHeadDim, (cuuint64_t)s.H, (cuuint64_t)s.N, (cuuint64_t)s.B};
  const cuuint64_t strides[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)s.H * kHeadDim, (cuuint64_t)s.N * s.H * kHeadDim};
  const cuuint32_t box[4] = {128, 1, 64, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SOL_OK : fail(SOL_ERR_LAUNCH, "cuTensorMapEncodeTiled (E4M3 BTHD) failed: %d", (int)r);
}

// E4M3 [BH][rows][128] bytes, 128 x 128 x 1 boxes (compressed keys / values of the FP8 path).
int encode_rows8(CUtensorMap* m, const void* base, int rows, const Shape& s) {
  const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows, (cuuint64_t)s.BH};
  const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows * kHeadDim};
  const cuuint32_t box[3] = {128, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SOL_OK : fail(SOL_ERR_LAUNCH, "cuTensorMapEncodeTiled (E4M3 rows) failed: %d", (int)r);
}

int check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SOL_ERR_LAUNCH, "%s: %s", what, cudaGetErrorString(e));
  return SOL_OK;
}

// Routing prefix shared by all entry points: summaries, threshold statistics, thresholds, bitmask.
int run_routing(DeviceState& d, const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                const Shape& s, const Work& w, float tau, int sink_start, int sink_tokens, bool anchors,
                bool diag, const sol_attn_options* opts, cudaStream_t st, int* launches,
                const Fp8Work* f8 = nullptr) {
  SinkSet sinks{};
  add_sink(s.N, sink_start, sink_tokens, &sinks);
  if (opts)
    for (int e = 0; e < opts->n_extra_sinks; ++e) add_sink(s.N, opts->extra_sink_start[e], opts->extra_sink_tokens[e], &sinks);
  if (cudaMemsetAsync(d.stats, 0, sizeof(unsigned long long), st) != cudaSuccess ||
      cudaMemsetAsync(d.stats + 1, 0xff, sizeof(unsigned long long), st) != cudaSuccess ||
      cudaMemsetAsync(d.stats + 2, 0, sizeof(unsigned long long), st) != cudaSuccess)
    return fail(SOL_ERR_LAUNCH, "stats reset failed");
  // every caller reaches the tensor-map encoder through here, so look it up here
  int rc = get_encode();
  if (rc) return rc;
  Work ww = w;
  ww.stats = d.stats;
  // FP8: the summary pass also quantises Q and K and takes the heads' max |V| (cleared here)
  if (f8 && cudaMemsetAsync(f8->vmax, 0, (size_t)s.BH * sizeof(unsigned int), st) != cudaSuccess)
    return fail(SOL_ERR_LAUNCH, "V maximum reset failed");
  if (anchors)
    launch_sol2_summaries(q, k, v, s, ww, st, f8);   // Sol-Attn2: the key groups come with the key means
  else
    launch_summary(q, k, v, s, ww, false, st, f8);
  launch_kstats(s, ww, st);
  launch_thresh(s, ww, tau, diag, st);
  CUtensorMap rmaps[4];
  if ((rc = encode_rows(&rmaps[0], w.qbar_hi, s.Nb, s)) || (rc = encode_rows(&rmaps[1], w.qbar_lo, s.Nb, s)) ||
      (rc = encode_rows(&rmaps[2], w.kbar_h, s.Nb, s)) || (rc = encode_rows(&rmaps[3], w.kbar_lo, s.Nb, s)))
    return rc;
  cudaError_t e = launch_route_tc(rmaps, s, ww, sinks, d.status, st);
  if (e != cudaSuccess) return fail(SOL_ERR_LAUNCH, "routing launch: %s", cudaGetErrorString(e));
  *launches += anchors ? 8 : 6;
  d.last_total_pairs = (long long)s.BH * s.Nb * s.Nb;
  return check_launch("routing kernels");
}

// Validates the options against the sequence length; sets *diag, *splits, *fp8 and *one_block.
int check_options(const sol_attn_options* o, int N, bool* diag, int* splits, bool* fp8, bool* one_block = nullptr) {
  *diag = false;
  *splits = 1;
  *fp8 = false;
  if (one_block) *one_block = false;
  if (!o) return SOL_OK;
  if (o->m_tile != 0 && o->m_tile != 64 && o->m_tile != 128)
    return fail(SOL_ERR_OPTION, "m_tile must be 0, 64 or 128 (got %d)", o->m_tile);
  if (o->m_tile == 64 && o->precision == SOL_PRECISION_FP8)
    return fail(SOL_ERR_OPTION, "m_tile 64 is available on the BF16 path only");
  if (one_block) *one_block = o->m_tile == 64;
  if (o->precision != SOL_PRECISION_BF16 && o->precision != SOL_PRECISION_FP8)
    return fail(SOL_ERR_OPTION, "unknown precision %d", o->precision);
  *fp8 = o->precision == SOL_PRECISION_FP8;
  if (o->kv_splits < 0 || o->kv_splits > SOL_MAX_KV_SPLITS)
    return fail(SOL_ERR_OPTION, "kv_splits must be in [0, %d]", SOL_MAX_KV_SPLITS);
  *splits = o->kv_splits > 1 ? o->kv_splits : 1;
  for (int r : o->reserved)
    if (r != 0) return fail(SOL_ERR_OPTION, "reserved option fields must be zero");
  if (o->thresh_type != SOL_THRESH_EXACT && o->thresh_type != SOL_THRESH_DIAG)
    return fail(SOL_ERR_OPTION, "unknown thresh_type %d", o->thresh_type);
  if (o->n_extra_sinks < 0 || o->n_extra_sinks > SOL_MAX_EXTRA_SINKS)
    return fail(SOL_ERR_OPTION, "n_extra_sinks must be in [0, %d]", SOL_MAX_EXTRA_SINKS);
  for (int e = 0; e < SOL_MAX_EXTRA_SINKS; ++e) {
    const bool used = e < o->n_extra_sinks;
    if (!used && (o->extra_sink_start[e] != 0 || o->extra_sink_tokens[e] != 0))
      return fail(SOL_ERR_OPTION, "unused extra sink slots must be zero");
    if (used && (o->extra_sink_start[e] < 0 || o->extra_sink_start[e] >= N || o->extra_sink_tokens[e] <= 0))
      return fail(SOL_ERR_OPTION, "extra sink %d needs 0 <= start < N and tokens > 0", e);
  }
  *diag = o->thresh_type == SOL_THRESH_DIAG;
  return SOL_OK;
}

int forward(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau, int sink_start,
            int sink_tokens, const sol_attn_options* opts, void* stream, bool sol2, bool fp8 = false) {
  int rc = validate(q, k, v, out, true, B, N, H, tau, sink_start, sink_tokens);
  if (rc) return rc;
  bool diag, opt_fp8, one_block;
  int splits;
  if ((rc = check_options(opts, N, &diag, &splits, &opt_fp8, &one_block))) return rc;
  fp8 = fp8 || opt_fp8;
  if (fp8 && one_block) return fail(SOL_ERR_OPTION, "m_tile 64 is available on the BF16 path only");
  if (sol2 && splits > 1) return fail(SOL_ERR_OPTION, "kv_splits > 1 is available for Sol-Attn only");
  if (fp8 && splits > 1) return fail(SOL_ERR_OPTION, "kv_splits > 1 is not available on the FP8 path");
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* d;
  int dev;
  if ((rc = device_state(&d, &dev))) return rc;
  if ((rc = get_encode())) return rc;
  const Shape s = make_shape(B, N, H);
  Work w;
  const size_t base = carve(s, sol2, nullptr, nullptr);
  const size_t rows_bh = (size_t)s.BH * s.QT * 128;
  const size_t part_o_bytes = splits > 1 ? (size_t)splits * rows_bh * 128 * 4 : 0;
  const size_t part_ml_bytes = splits > 1 ? (size_t)splits * rows_bh * 2 * 4 : 0;
  const size_t fp8_bytes = fp8 ? carve_fp8(s, nullptr, nullptr) : 0;
  if ((rc = ensure_workspace(*d, base + part_o_bytes + part_ml_bytes + fp8_bytes))) return rc;
  carve(s, sol2, static_cast<char*>(d->ws), &w);
  Fp8Work f8{};
  if (fp8) carve_fp8(s, static_cast<char*>(d->ws) + base + part_o_bytes + part_ml_bytes, &f8);
  float* part_o = splits > 1 ? reinterpret_cast<float*>(static_cast<char*>(d->ws) + base) : nullptr;
  float* part_ml = splits > 1 ? reinterpret_cast<float*>(static_cast<char*>(d->ws) + base + part_o_bytes) : nullptr;
  w.stats = d->stats;

  CUtensorMap maps[5];
  if (fp8) {
    const int nbp = fp8_rows_padded(s);
    if ((rc = encode_bthd8(&maps[0], f8.q8, s)) || (rc = encode_bthd8(&maps[1], f8.k8, s)) ||
        (rc = encode_bthd8(&maps[2], f8.v8, s)) || (rc = encode_rows8(&maps[3], f8.kbar8, nbp, s)) ||
        (rc = encode_rows8(&maps[4], f8.vbar8, nbp, s)))
      return rc;
  } else if ((rc = encode_bthd(&maps[0], q, s)) || (rc = encode_bthd(&maps[1], k, s)) ||
             (rc = encode_bthd(&maps[2], v, s)) || (rc = encode_pooled(&maps[3], w.kbar_h, s)) ||
             (rc = encode_pooled(&maps[4], w.vbar_h, s))) {
    return rc;
  }

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamWaitEvent(st, d->done, 0) != cudaSuccess) return fail(SOL_ERR_LAUNCH, "cudaStreamWaitEvent failed");
  int launches = 0;
  const auto* qh = static_cast<const __nv_bfloat16*>(q);
  const auto* kh = static_cast<const __nv_bfloat16*>(k);
  const auto* vh = static_cast<const __nv_bfloat16*>(v);
  if ((rc = run_routing(*d, qh, kh, vh, s, w, tau, sink_start, sink_tokens, sol2, diag, opts, st, &launches,
                        fp8 ? &f8 : nullptr)))
    return rc;
  if (sol2) {
    CUtensorMap tmaps[3];
    if ((rc = encode_rows(&tmaps[0], w.qanchor_h, s.Na, s)) || (rc = encode_rows(&tmaps[1], w.gk_h, 2 * s.Nb, s)) ||
        (rc = encode_rows(&tmaps[2], w.gv_h, 2 * s.Nb, s)))
      return rc;
    cudaError_t te = launch_tail_tc(tmaps, s, w, d->status, st);
    if (te != cudaSuccess) return fail(SOL_ERR_LAUNCH, "Sol-Attn2 tail launch: %s", cudaGetErrorString(te));
    launches += 1;
    if ((rc = check_launch("Sol-Attn2 tail kernels"))) return rc;
  }
  if (fp8) {
    launch_quant_fp8(vh, s, w, f8, st);
    launches += 2;
    if ((rc = check_launch("FP8 quantisation kernels"))) return rc;
  }
  FwdParams p{};
  p.N = N;
  p.H = H;
  p.Nb = s.Nb;
  p.Nw = s.Nw;
  p.Na = s.Na;
  p.QT = s.QT;
  p.mask = w.mask;
  p.qt_begin = 0;
  p.unit_blocks = one_block ? 1 : 2;
  p.qt_count = one_block ? s.Nb : s.QT;   // work units per (b, h)
  p.row_lo = 0;
  p.row_hi = N;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.status = d->status;
  p.qanchor = w.qanchor;
  p.tail_logz = w.tail_logz;
  p.tail_mu = w.tail_mu;
  p.tail_nu = w.tail_nu;
  p.kv_splits = splits;
  p.part_o = part_o;
  p.part_ml = part_ml;
  p.part_rows_bh = rows_bh;
  const int grid = s.BH * p.qt_count * splits;
  if (g_unit_timing && !fp8) {
    const size_t units = (size_t)grid;
    if (d->unit_cap < units) {
      if (d->unit_buf) {
        cudaDeviceSynchronize();
        cudaFree(d->unit_buf);
      }
      d->unit_buf = nullptr;
      d->unit_cap = 0;
      if (cudaMalloc(&d->unit_buf, units * 3 * sizeof(unsigned long long)) != cudaSuccess) {
        cudaGetLastError();
        return fail(SOL_ERR_ALLOC, "unit timing buffer allocation failed");
      }
      d->unit_cap = units;
    }
    p.unit_times = d->unit_buf;
    d->last_units = (int)units;
  }
  const int slot = d->timed_calls % DeviceState::kRing;
  if (g_timing) {
    if (!d->t0[slot] && (cudaEventCreate(&d->t0[slot]) != cudaSuccess || cudaEventCreate(&d->t1[slot]) != cudaSuccess))
      return fail(SOL_ERR_LAUNCH, "timing event creation failed");
    cudaEventRecord(d->t0[slot], st);
  }
  cudaError_t e;
  if (fp8) {
    const Fp8Params fp{f8.sq, f8.sk, f8.skbar, f8.sv, fp8_rows_padded(s) / 64};
    e = launch_attn_fwd_fp8(maps, p, fp, s.BH * s.QT, sol2, st);
  } else {
    e = launch_attn_fwd(maps, p, grid, sol2, st);
  }
  if (e != cudaSuccess) return fail(SOL_ERR_LAUNCH, "fused attention launch: %s", cudaGetErrorString(e));
  if (splits > 1) {
    launch_splitkv_combine(s, splits, part_o, part_ml, p.out, 0, N, st);
    launches += 1;
    if ((rc = check_launch("split-KV combine"))) return rc;
  }
  if (g_timing) {
    cudaEventRecord(d->t1[slot], st);
    ++d->timed_calls;
  }
  launches += 1;
  cudaEventRecord(d->done, st);
  d->last_stream = st;
  d->last_launches = launches;
  g_last_device = dev;
  return SOL_OK;
}

// Exact (dense) attention for the query tokens [q_start, q_start + q_tokens): the fused kernel
// over the query tiles that cover them, every key block marked exact for those query blocks, and
// only rows inside the range written.
int dense_rows(const void* q, const void* k, const void* v, void* out, int B, int N, int H, int q_start, int q_tokens,
               void* stream) {
  int rc = validate(q, k, v, out, true, B, N, H, 1.0f, -1, 0);
  if (rc) return rc;
  if (q_tokens > 0 && q_start >= N) return fail(SOL_ERR_SINK, "q_start (%d) must be < N (%d)", q_start, N);
  long long r0 = q_start >= 0 ? q_start : (long long)N - q_tokens;
  long long r1 = r0 + (q_tokens > 0 ? q_tokens : 0);
  if (r0 < 0) r0 = 0;
  if (r1 > N) r1 = N;
  if (r1 <= r0) return SOL_OK;   // no rows: nothing to do
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* d;
  int dev;
  if ((rc = device_state(&d, &dev))) return rc;
  if ((rc = get_encode())) return rc;
  const Shape s = make_shape(B, N, H);
  Work w;
  if ((rc = ensure_workspace(*d, carve(s, false, nullptr, nullptr)))) return rc;
  carve(s, false, static_cast<char*>(d->ws), &w);
  w.stats = d->stats;
  // the kernel's pooled-tile maps must be valid descriptors; no pooled tile is loaded here
  CUtensorMap maps[5];
  if ((rc = encode_bthd(&maps[0], q, s)) || (rc = encode_bthd(&maps[1], k, s)) || (rc = encode_bthd(&maps[2], v, s)) ||
      (rc = encode_pooled(&maps[3], w.kbar_h, s)) || (rc = encode_pooled(&maps[4], w.vbar_h, s)))
    return rc;
  const int qt0 = (int)(r0 / kBlock) / 2, qt1 = (int)((r1 - 1) / kBlock) / 2;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamWaitEvent(st, d->done, 0) != cudaSuccess) return fail(SOL_ERR_LAUNCH, "cudaStreamWaitEvent failed");
  launch_dense_mask(s, w, 2 * qt0, std::min(2 * qt1 + 1, s.Nb - 1), st);
  FwdParams p{};
  p.N = N;
  p.H = H;
  p.Nb = s.Nb;
  p.Nw = s.Nw;
  p.Na = s.Na;
  p.QT = s.QT;
  p.mask = w.mask;
  p.qt_begin = qt0;
  p.qt_count = qt1 - qt0 + 1;
  p.row_lo = (int)r0;
  p.row_hi = (int)r1;
  p.kv_splits = 1;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.status = d->status;
  cudaError_t e = launch_attn_fwd(maps, p, s.BH * p.qt_count, false, st);
  if (e != cudaSuccess) return fail(SOL_ERR_LAUNCH, "fused attention launch: %s", cudaGetErrorString(e));
  if ((rc = check_launch("dense rows"))) return rc;
  cudaEventRecord(d->done, st);
  d->last_stream = st;
  d->last_launches = 2;
  g_last_device = dev;
  return SOL_OK;
}

// Self-test of the bounded-wait path: one thread waits on an mbarrier whose phase never completes
// (nothing arrives on it), so the wait runs out after kWaitLimitNs and records a timeout in the
// device status word exactly as a stalled pipeline stage would.  No trap, no fault: the kernel
// returns normally and the context stays usable.
__global__ void wait_timeout_selftest_kernel(int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &abort_flag)) atomicExch(status, kDevTimeout);
}

}  // namespace

void set_last_error(const char* msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }

}  // namespace sol

namespace sol {
namespace {

// The host-buffer entry points: heads are independent problems, so the (b, head-chunk) slices are
// pipelined: the strided copy of slice c + 1 into the device overlaps the attention of slice c and
// the copy of slice c - 1 back to the host.
int host_pipeline(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                  int sink_start, int sink_tokens, const sol_attn_options* opts, int heads_per_chunk, bool sol2) {
  if (!q || !k || !v || !out) return fail(SOL_ERR_NULL, "q, k, v and out must be non-NULL");
  if (B <= 0 || N <= 0 || H <= 0) return fail(SOL_ERR_SHAPE, "B, N, H must be positive (got %d, %d, %d)", B, N, H);
  if ((long long)B * N * H * kHeadDim > (1ll << 40)) return fail(SOL_ERR_SHAPE, "sizes out of the supported range");
  if (heads_per_chunk < 0) return fail(SOL_ERR_SHAPE, "heads_per_chunk must be >= 0");
  const int hc = heads_per_chunk > 0 ? std::min(heads_per_chunk, H) : std::max(1, (H + 15) / 16);
  const size_t row = (size_t)H * kHeadDim * 2;            // bytes per token of the host tensors
  const size_t crow = (size_t)hc * kHeadDim * 2;          // bytes per token of one slice
  const size_t slice = (size_t)N * crow;
  std::lock_guard<std::mutex> hlock(g_host_mu);
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return fail(SOL_ERR_DEVICE, "no current CUDA device");
  HostPipe& hp = g_pipe[dev];
  if (!hp.ready) {
    bool okc = cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking) == cudaSuccess &&
               cudaStreamCreateWithFlags(&hp.comp, cudaStreamNonBlocking) == cudaSuccess &&
               cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking) == cudaSuccess;
    for (int i = 0; i < 2 && okc; ++i)
      okc = cudaEventCreateWithFlags(&hp.in_done[i], cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&hp.comp_done[i], cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&hp.out_done[i], cudaEventDisableTiming) == cudaSuccess;
    if (!okc) {
      cudaGetLastError();
      return fail(SOL_ERR_DEVICE, "stream / event creation failed");
    }
    hp.ready = true;
  }
  const size_t need = 4 * align_up(slice, 256);
  if (hp.buf_bytes < need) {
    for (int i = 0; i < 2; ++i) {
      if (hp.buf[i]) {
        cudaStreamSynchronize(hp.out);
        cudaFree(hp.buf[i]);
      }
      hp.buf[i] = nullptr;
    }
    hp.buf_bytes = 0;
    for (int i = 0; i < 2; ++i)
      if (cudaMalloc(&hp.buf[i], need) != cudaSuccess) {
        cudaGetLastError();
        return fail(SOL_ERR_ALLOC, "staging buffers of %zu bytes failed", 2 * need);
      }
    hp.buf_bytes = need;
  }
  const int chunks_per_b = (H + hc - 1) / hc;
  const int nchunks = B * chunks_per_b;
  int rc = SOL_OK;
  for (int c = 0; c < nchunks && rc == SOL_OK; ++c) {
    const int i = c & 1;
    const int b = c / chunks_per_b, h0 = (c % chunks_per_b) * hc, hn = std::min(hc, H - h0);
    const size_t cw = (size_t)hn * kHeadDim * 2;          // bytes per token of this slice
    char* base = hp.buf[i];
    char* dq = base;
    char* dk = base + align_up(slice, 256);
    char* dv = base + 2 * align_up(slice, 256);
    char* dout = base + 3 * align_up(slice, 256);
    const size_t hoff = ((size_t)b * N * H + h0) * kHeadDim * 2;
    // slice c reuses the buffers of slice c - 2: its compute read them and its output left them
    if (c >= 2 && (cudaStreamWaitEvent(hp.in, hp.comp_done[i], 0) != cudaSuccess ||
                   cudaStreamWaitEvent(hp.in, hp.out_done[i], 0) != cudaSuccess)) {
      rc = fail(SOL_ERR_LAUNCH, "stream ordering failed");
      break;
    }
    if (cudaMemcpy2DAsync(dq, cw, static_cast<const char*>(q) + hoff, row, cw, N, cudaMemcpyHostToDevice, hp.in) != cudaSuccess ||
        cudaMemcpy2DAsync(dk, cw, static_cast<const char*>(k) + hoff, row, cw, N, cudaMemcpyHostToDevice, hp.in) != cudaSuccess ||
        cudaMemcpy2DAsync(dv, cw, static_cast<const char*>(v) + hoff, row, cw, N, cudaMemcpyHostToDevice, hp.in) != cudaSuccess ||
        cudaEventRecord(hp.in_done[i], hp.in) != cudaSuccess || cudaStreamWaitEvent(hp.comp, hp.in_done[i], 0) != cudaSuccess) {
      rc = fail(SOL_ERR_LAUNCH, "host-to-device copy failed: %s", cudaGetErrorString(cudaGetLastError()));
      break;
    }
    rc = forward(dq, dk, dv, dout, 1, N, hn, tau, sink_start, sink_tokens, opts, hp.comp, sol2);
    if (rc) break;
    if (cudaEventRecord(hp.comp_done[i], hp.comp) != cudaSuccess || cudaStreamWaitEvent(hp.out, hp.comp_done[i], 0) != cudaSuccess ||
        cudaMemcpy2DAsync(static_cast<char*>(out) + hoff, row, dout, cw, cw, N, cudaMemcpyDeviceToHost, hp.out) != cudaSuccess ||
        cudaEventRecord(hp.out_done[i], hp.out) != cudaSuccess) {
      rc = fail(SOL_ERR_LAUNCH, "device-to-host copy failed: %s", cudaGetErrorString(cudaGetLastError()));
      break;
    }
  }
  // the call returns with the output in host memory (or after an error, with nothing in flight)
  const bool synced = cudaStreamSynchronize(hp.in) == cudaSuccess && cudaStreamSynchronize(hp.comp) == cudaSuccess &&
                      cudaStreamSynchronize(hp.out) == cudaSuccess;
  if (rc == SOL_OK && !synced) rc = fail(SOL_ERR_LAUNCH, "synchronisation failed: %s", cudaGetErrorString(cudaGetLastError()));
  return rc;
}

}  // namespace
}  // namespace sol

using namespace sol;

extern "C" {


int sol_attn_fwd(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                 int sink_start, int sink_tokens, void* stream) {
  g_err[0] = 0;
  return forward(q, k, v, out, B, N, H, tau, sink_start, sink_tokens, nullptr, stream, false);
}

int sol_attn2_fwd(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                  int sink_start, int sink_tokens, void* stream) {
  g_err[0] = 0;
  return forward(q, k, v, out, B, N, H, tau, sink_start, sink_tokens, nullptr, stream, true);
}

int sol_attn_fwd_ex(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                    int sink_start, int sink_tokens, const sol_attn_options* opts, void* stream) {
  g_err[0] = 0;
  return forward(q, k, v, out, B, N, H, tau, sink_start, sink_tokens, opts, stream, false);
}

int sol_attn2_fwd_ex(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                     int sink_start, int sink_tokens, const sol_attn_options* opts, void* stream) {
  g_err[0] = 0;
  return forward(q, k, v, out, B, N, H, tau, sink_start, sink_tokens, opts, stream, true);
}

const char* sol_attn_last_error(void) { return g_err; }

int sol_attn_get_device_status(void* stream) {
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* d;
  int dev;
  int rc = device_state(&d, &dev);
  if (rc) return rc;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return fail(SOL_ERR_LAUNCH, "stream synchronisation failed: %s", cudaGetErrorString(cudaGetLastError()));
  int h = 0;
  if (cudaMemcpy(&h, d->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemset(d->status, 0, sizeof(int)) != cudaSuccess)
    return fail(SOL_ERR_LAUNCH, "status read failed");
  if (h == kDevTimeout) return fail(SOL_ERR_TIMEOUT, "a bounded wait inside a kernel ran out");
  if (h == kDevMisaligned) return fail(SOL_ERR_LAUNCH, "shared memory window misaligned; the kernel did not run");
  if (h == kDevBounds) return fail(SOL_ERR_LAUNCH, "a bounds check of the debug build failed (access skipped)");
  return SOL_OK;
}

int sol_attn_debug_route_ex(const void* q, const void* k, int B, int N, int H, float tau, int sink_start,
                            int sink_tokens, const sol_attn_options* opts, unsigned char* mask, float* thresh,
                            void* stream) {
  g_err[0] = 0;
  int rc = validate(q, k, nullptr, nullptr, false, B, N, H, tau, sink_start, sink_tokens);
  if (rc) return rc;
  bool diag;
  int splits;
  bool fp8_unused;
  if ((rc = check_options(opts, N, &diag, &splits, &fp8_unused))) return rc;
  if (!mask) return fail(SOL_ERR_NULL, "mask must be non-NULL");
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* d;
  int dev;
  if ((rc = device_state(&d, &dev))) return rc;
  const Shape s = make_shape(B, N, H);
  Work w;
  if ((rc = ensure_workspace(*d, carve(s, false, nullptr, nullptr)))) return rc;
  carve(s, false, static_cast<char*>(d->ws), &w);
  w.stats = d->stats;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaStreamWaitEvent(st, d->done, 0);
  int launches = 0;
  // the summary kernel reads v as well; pass k, whose summaries are simply discarded
  if ((rc = run_routing(*d, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                        static_cast<const __nv_bfloat16*>(k), s, w, tau, sink_start, sink_tokens, false, diag, opts,
                        st, &launches)))
    return rc;
  launch_expand_mask(s, w, mask, st);
  if (thresh) cudaMemcpyAsync(thresh, w.thresh, (size_t)s.BH * s.Nb * sizeof(float), cudaMemcpyDeviceToDevice, st);
  if ((rc = check_launch("route introspection"))) return rc;
  cudaEventRecord(d->done, st);
  d->last_stream = st;
  d->last_launches = launches + 1;
  g_last_device = dev;
  return SOL_OK;
}

int sol_attn_debug_route(const void* q, const void* k, int B, int N, int H, float tau, int sink_start,
                         int sink_tokens, unsigned char* mask, float* thresh, void* stream) {
  return sol_attn_debug_route_ex(q, k, B, N, H, tau, sink_start, sink_tokens, nullptr, mask, thresh, stream);
}

int sol_attn_last_stats(long long* exact_pairs, long long* total_pairs, int* min_row, int* max_row) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_last_device < 0) return fail(SOL_ERR_LAUNCH, "no call has run yet");
  DeviceState& d = g_dev[g_last_device];
  int cur = -1;
  cudaGetDevice(&cur);
  cudaSetDevice(g_last_device);
  unsigned long long h[3] = {0, 0, 0};
  cudaError_t e = cudaStreamSynchronize(d.last_stream);
  if (e == cudaSuccess) e = cudaMemcpy(h, d.stats, sizeof(h), cudaMemcpyDeviceToHost);
  cudaSetDevice(cur);
  if (e != cudaSuccess) return fail(SOL_ERR_LAUNCH, "stats read failed: %s", cudaGetErrorString(e));
  if (exact_pairs) *exact_pairs = (long long)h[0];
  if (total_pairs) *total_pairs = d.last_total_pairs;
  if (min_row) *min_row = (int)h[1];
  if (max_row) *max_row = (int)h[2];
  return SOL_OK;
}

int sol_attn_set_kernel_timing(int enable) {
  std::lock_guard<std::mutex> lock(g_mu);
  g_timing = enable != 0;
  if (g_timing)
    for (auto& d : g_dev) d.timed_calls = 0;
  return SOL_OK;
}

static float kernel_ms_sum_locked(int n) {
  if (g_last_device < 0) return -1.f;
  DeviceState& d = g_dev[g_last_device];
  if (n <= 0 || n > d.timed_calls || n > DeviceState::kRing) return -1.f;
  double total = 0.0;
  for (int i = d.timed_calls - n; i < d.timed_calls; ++i) {
    const int slot = i % DeviceState::kRing;
    float ms = -1.f;
    if (cudaEventSynchronize(d.t1[slot]) != cudaSuccess || cudaEventElapsedTime(&ms, d.t0[slot], d.t1[slot]) != cudaSuccess)
      return -1.f;
    total += ms;
  }
  return (float)total;
}

int sol_attn_set_unit_timing(int enable) {
  std::lock_guard<std::mutex> lock(g_mu);
  g_unit_timing = enable != 0;
  return SOL_OK;
}

int sol_attn_last_unit_times(unsigned long long* host, int max_units, int* units) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!host || !units) return fail(SOL_ERR_NULL, "host and units must be non-NULL");
  if (g_last_device < 0) return fail(SOL_ERR_LAUNCH, "no call has run yet");
  DeviceState& d = g_dev[g_last_device];
  if (!d.unit_buf || d.last_units <= 0) return fail(SOL_ERR_LAUNCH, "no fused launch ran with unit timing enabled");
  int cur = -1;
  cudaGetDevice(&cur);
  cudaSetDevice(g_last_device);
  const int n = std::min(max_units, d.last_units);
  cudaError_t e = cudaStreamSynchronize(d.last_stream);
  if (e == cudaSuccess && n > 0) e = cudaMemcpy(host, d.unit_buf, (size_t)n * 3 * sizeof(unsigned long long), cudaMemcpyDeviceToHost);
  cudaSetDevice(cur);
  if (e != cudaSuccess) return fail(SOL_ERR_LAUNCH, "unit times read failed: %s", cudaGetErrorString(e));
  *units = d.last_units;
  return SOL_OK;
}

float sol_attn_last_kernel_ms(void) {
  std::lock_guard<std::mutex> lock(g_mu);
  return kernel_ms_sum_locked(1);
}

float sol_attn_kernel_ms_sum(int n) {
  std::lock_guard<std::mutex> lock(g_mu);
  return kernel_ms_sum_locked(n);
}

int sol_attn_last_launch_count(void) {
  std::lock_guard<std::mutex> lock(g_mu);
  return g_last_device < 0 ? 0 : g_dev[g_last_device].last_launches;
}

void sol_attn_release_workspace(void) {
  std::lock_guard<std::mutex> hlock(g_host_mu);
  std::lock_guard<std::mutex> lock(g_mu);
  int cur = -1;
  cudaGetDevice(&cur);
  for (int i = 0; i < kMaxDevices; ++i) {
    DeviceState& d = g_dev[i];
    HostPipe& hp = g_pipe[i];
    if (!d.ws && !hp.buf[0]) continue;
    cudaSetDevice(i);
    cudaDeviceSynchronize();
    if (d.ws) cudaFree(d.ws);
    d.ws = nullptr;
    d.ws_bytes = 0;
    for (int j = 0; j < 2; ++j) {
      if (hp.buf[j]) cudaFree(hp.buf[j]);
      hp.buf[j] = nullptr;
    }
    hp.buf_bytes = 0;
  }
  if (cur >= 0) cudaSetDevice(cur);
}

int sol_attn_dense_rows(const void* q, const void* k, const void* v, void* out, int B, int N, int H, int q_start,
                        int q_tokens, void* stream) {
  g_err[0] = 0;
  return dense_rows(q, k, v, out, B, N, H, q_start, q_tokens, stream);
}

int sol_attn_selftest_wait_timeout(void* stream) {
  g_err[0] = 0;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState* d;
  int dev;
  int rc = device_state(&d, &dev);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  wait_timeout_selftest_kernel<<<1, 32, 0, st>>>(d->status);
  if ((rc = check_launch("wait-timeout self-test"))) return rc;
  d->last_stream = st;
  return SOL_OK;
}

int sol_attn_fwd_varlen(const void* q, const void* k, const void* v, void* out, const int* cu_seqlens, int nseq,
                        int H, float tau, int sink_start, int sink_tokens, const sol_attn_options* opts, void* stream) {
  g_err[0] = 0;
  if (!cu_seqlens) return fail(SOL_ERR_NULL, "cu_seqlens must be non-NULL");
  if (nseq <= 0 || H <= 0) return fail(SOL_ERR_SHAPE, "nseq and H must be positive");
  if (cu_seqlens[0] != 0) return fail(SOL_ERR_SHAPE, "cu_seqlens[0] must be 0");
  for (int i = 0; i < nseq; ++i)
    if (cu_seqlens[i + 1] < cu_seqlens[i]) return fail(SOL_ERR_SHAPE, "cu_seqlens must be non-decreasing");
  // every sequence must satisfy the single-sequence rules (a sink range starts inside each one)
  for (int i = 0; i < nseq; ++i) {
    const int n = cu_seqlens[i + 1] - cu_seqlens[i];
    if (n > 0 && sink_tokens > 0 && sink_start >= n)
      return fail(SOL_ERR_SINK, "sink_start (%d) must be < the length of sequence %d (%d)", sink_start, i, n);
  }
  const size_t row = (size_t)H * 128 * 2;   // bytes per token
  for (int i = 0; i < nseq; ++i) {
    const int n = cu_seqlens[i + 1] - cu_seqlens[i];
    if (n == 0) continue;
    const size_t off = (size_t)cu_seqlens[i] * row;
    const int rc = forward(static_cast<const char*>(q) + off, static_cast<const char*>(k) + off,
                           static_cast<const char*>(v) + off, static_cast<char*>(out) + off, 1, n, H, tau, sink_start,
                           sink_tokens, opts, stream, false);
    if (rc) return rc;
  }
  return SOL_OK;
}

int sol_attn_fwd_host(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                      int sink_start, int sink_tokens, const sol_attn_options* opts, int heads_per_chunk) {
  g_err[0] = 0;
  return host_pipeline(q, k, v, out, B, N, H, tau, sink_start, sink_tokens, opts, heads_per_chunk, false);
}

int sol_attn2_fwd_host(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                       int sink_start, int sink_tokens, const sol_attn_options* opts, int heads_per_chunk) {
  g_err[0] = 0;
  return host_pipeline(q, k, v, out, B, N, H, tau, sink_start, sink_tokens, opts, heads_per_chunk, true);
}

int sol_attn_fwd_fp8(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                     int sink_start, int sink_tokens, const sol_attn_options* opts, void* stream) {
  return forward(q, k, v, out, B, N, H, tau, sink_start, sink_tokens, opts, stream, false, true);
}

int sol_attn2_fwd_fp8(const void* q, const void* k, const void* v, void* out, int B, int N, int H, float tau,
                      int sink_start, int sink_tokens, const sol_attn_options* opts, void* stream) {
  return forward(q, k, v, out, B, N, H, tau, sink_start, sink_tokens, opts, stream, true, true);
}

int sol_attn_expcast_host(const float* x, int n, float fs, float pivot, unsigned int* words) {
  if (!x || !words) return fail(SOL_ERR_NULL, "x and words must be non-NULL");
  if (n < 0 || n % 4) return fail(SOL_ERR_SHAPE, "n must be a non-negative multiple of 4 (got %d)", n);
  if (!(fs > 0.f) || !std::isfinite(fs) || !std::isfinite(pivot) || pivot != std::floor(pivot))
    return fail(SOL_ERR_OPTION, "fs must be positive and finite and pivot a finite integer");
  const float c0 = kExpCastOffset - 8.0f * pivot;
  for (int i = 0; i < n; i += 4)
    words[i / 4] = pack_codes4(expcast_code_f32(x[i], 8.0f * fs, c0), expcast_code_f32(x[i + 1], 8.0f * fs, c0),
                               expcast_code_f32(x[i + 2], 8.0f * fs, c0), expcast_code_f32(x[i + 3], 8.0f * fs, c0));
  return SOL_OK;
}

int sol_attn_quot448_host(const float* x, int n, float m, float* q) {
  if (!x || !q) return fail(SOL_ERR_NULL, "x and q must be non-NULL");
  if (n < 0) return fail(SOL_ERR_SHAPE, "n must be non-negative (got %d)", n);
  if (!(m > 0.f) || !std::isfinite(m)) return fail(SOL_ERR_OPTION, "m must be positive and finite");
  const Quot448 c = quot448_setup(m);
  for (int i = 0; i < n; ++i) q[i] = quot448(x[i], c);
  return SOL_OK;
}

void sol_attn_set_workspace_limit(size_t bytes) {
  std::lock_guard<std::mutex> lock(g_mu);
  g_ws_limit = bytes;
}

}  // extern "C"
