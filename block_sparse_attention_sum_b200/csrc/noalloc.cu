// Allocation-free variant of sol_attn_fwd for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they run attention: code inside a memory
// pool that forbids outside allocations, an embedded runtime that has reserved all device memory up
// front, or a process whose allocator must not be touched while other work holds the device.  For
// them, sol_attn_fwd_noalloc runs the same kernels as sol_attn_fwd, but its workspace is a fixed
// region of device memory declared at file scope in this library (kNoAllocScratchBytes, 64 MiB),
// plus two small status / statistics words, all of which every GPU that loads the library keeps
// until the process exits.  The call itself never allocates or frees device memory.
//
// Host code cannot use the name of a __device__ array as a device address (it is a host-side
// shadow); the device address is looked up with cudaGetSymbolAddress once per device, on the first
// call made while that device is current, and passed to the kernels.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <mutex>

#include "attn_fwd.cuh"
#include "common.cuh"
#include "ptx.cuh"
#include "sol_attn.h"

namespace sol {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
__device__ __align__(16) int g_noalloc_status[4];
__device__ __align__(16) unsigned long long g_noalloc_stats[4];

constexpr int kMaxDev = 64;
struct NoAllocDevice {
  bool ready = false;
  unsigned char* scratch = nullptr;
  int* status = nullptr;
  unsigned long long* stats = nullptr;
};
NoAllocDevice g_na[kMaxDev];
std::mutex g_na_mu;

// errors are reported through sol_attn_last_error() like every other entry point
int na_fail(int code, const char* msg) {
  set_last_error(msg);
  return code;
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// Same buffer set and order as the pooled workspace of sol_attn_fwd.
size_t na_carve(const Shape& s, unsigned char* base, Work* w) {
  size_t off = 0;
  auto take = [&](size_t bytes) {
    unsigned char* p = base ? base + off : nullptr;
    off = up256(off + bytes);
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
  if (w) *w = t;
  return off;
}

// Looks up, once per device and with that device current, the device addresses of the file-scope
// buffers.  cudaGetSymbolAddress also loads this file's module on the device if it is not loaded
// yet (lazy module loading), and that load is when the driver reserves the 64 MiB region.
// Caller holds g_na_mu.
int na_setup(NoAllocDevice** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return na_fail(SOL_ERR_DEVICE, "no current CUDA device");
  NoAllocDevice& d = g_na[dev];
  if (!d.ready) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess || major != 10 ||
        minor != 0)
      return na_fail(SOL_ERR_DEVICE, "the current device is not an sm_100 (B200-class) GPU");
    void* a = nullptr;
    void* b = nullptr;
    void* c = nullptr;
    if (cudaGetSymbolAddress(&a, g_noalloc_scratch) != cudaSuccess ||
        cudaGetSymbolAddress(&b, g_noalloc_status) != cudaSuccess ||
        cudaGetSymbolAddress(&c, g_noalloc_stats) != cudaSuccess || !a || !b || !c) {
      cudaGetLastError();
      return na_fail(SOL_ERR_DEVICE, "cudaGetSymbolAddress failed for the scratch region");
    }
    d.scratch = static_cast<unsigned char*>(a);
    d.status = static_cast<int*>(b);
    d.stats = static_cast<unsigned long long*>(c);
    d.ready = true;
  }
  *out = &d;
  return SOL_OK;
}

int na_encode(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap* m, const void* base, int rank,
              const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box) {
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SOL_OK : na_fail(SOL_ERR_LAUNCH, "cuTensorMapEncodeTiled failed");
}

}  // namespace
}  // namespace sol

using namespace sol;

extern "C" int sol_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out, int B, int N, int H,
                                    float tau, int sink_start, int sink_tokens, void* stream) {
  set_last_error("");
  if (!q || !k || !v || !out) return na_fail(SOL_ERR_NULL, "q, k, v and out must be non-NULL");
  if (B <= 0 || N <= 0 || H <= 0) return na_fail(SOL_ERR_SHAPE, "B, N, H must be positive");
  if ((long long)B * N * H * kHeadDim > (1ll << 40) || (long long)B * H > (1ll << 24))
    return na_fail(SOL_ERR_SHAPE, "sizes out of the supported range");
  if (!std::isfinite(tau)) return na_fail(SOL_ERR_TAU, "tau must be finite");
  if (sink_tokens > 0 && sink_start >= N) return na_fail(SOL_ERR_SINK, "sink_start must be < N");
  const uintptr_t mis = reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
                        reinterpret_cast<uintptr_t>(v) | reinterpret_cast<uintptr_t>(out);
  if (mis & 15u) return na_fail(SOL_ERR_ALIGN, "tensor pointers must be 16-byte aligned");
  const size_t bytes = (size_t)B * N * H * kHeadDim * 2;
  auto ov = [&](const void* a, const void* b2) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b2);
    return x < y + bytes && y < x + bytes;
  };
  if (ov(out, q) || ov(out, k) || ov(out, v)) return na_fail(SOL_ERR_ALIGN, "out must not overlap q, k or v");

  const Shape s = make_shape(B, N, H);
  const size_t need = na_carve(s, nullptr, nullptr);
  if (need > kNoAllocScratchBytes) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "this shape needs %zu bytes of scratch; the allocation-free entry point has %zu (use sol_attn_fwd)", need,
             kNoAllocScratchBytes);
    return na_fail(SOL_ERR_SHAPE, msg);
  }

  std::lock_guard<std::mutex> lock(g_na_mu);
  NoAllocDevice* dp = nullptr;
  int rc0 = na_setup(&dp);
  if (rc0) return rc0;
  NoAllocDevice& d = *dp;

  void* fn = nullptr;
  cudaDriverEntryPointQueryResult qr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) != cudaSuccess ||
      qr != cudaDriverEntryPointSuccess || !fn)
    return na_fail(SOL_ERR_DEVICE, "cuTensorMapEncodeTiled is unavailable");
  auto enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);

  Work w;
  na_carve(s, d.scratch, &w);
  w.stats = d.stats;

  CUtensorMap maps[9];
  const cuuint64_t dims4[4] = {(cuuint64_t)kHeadDim, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  const cuuint64_t str4[3] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)H * kHeadDim * 2, (cuuint64_t)N * H * kHeadDim * 2};
  const cuuint32_t box4[4] = {64, 1, 64, 1};
  const cuuint64_t dims3[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)s.Nb, (cuuint64_t)s.BH};
  const cuuint64_t str3[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)s.Nb * kHeadDim * 2};
  const cuuint32_t box3[3] = {64, 128, 1};
  int rc;
  if ((rc = na_encode(enc, &maps[0], q, 4, dims4, str4, box4)) || (rc = na_encode(enc, &maps[1], k, 4, dims4, str4, box4)) ||
      (rc = na_encode(enc, &maps[2], v, 4, dims4, str4, box4)) ||
      (rc = na_encode(enc, &maps[3], w.kbar_h, 3, dims3, str3, box3)) ||
      (rc = na_encode(enc, &maps[4], w.vbar_h, 3, dims3, str3, box3)) ||
      (rc = na_encode(enc, &maps[5], w.qbar_hi, 3, dims3, str3, box3)) ||
      (rc = na_encode(enc, &maps[6], w.qbar_lo, 3, dims3, str3, box3)) ||
      (rc = na_encode(enc, &maps[7], w.kbar_h, 3, dims3, str3, box3)) ||
      (rc = na_encode(enc, &maps[8], w.kbar_lo, 3, dims3, str3, box3)))
    return rc;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the routing statistics accumulate atomically: clear them (min row starts at all ones)
  if (cudaMemsetAsync(d.stats, 0, sizeof(unsigned long long), st) != cudaSuccess ||
      cudaMemsetAsync(d.stats + 1, 0xff, sizeof(unsigned long long), st) != cudaSuccess ||
      cudaMemsetAsync(d.stats + 2, 0, sizeof(unsigned long long), st) != cudaSuccess)
    return na_fail(SOL_ERR_LAUNCH, "statistics reset failed");

  SinkSet sinks{};
  if (sink_tokens > 0) {
    long long start = sink_start >= 0 ? sink_start : (long long)N - sink_tokens;
    long long end = start + sink_tokens;
    if (start < 0) start = 0;
    if (end > N) end = N;
    if (end > start) {
      sinks.b0[0] = (int)(start / kBlock);
      sinks.b1[0] = (int)((end - 1) / kBlock);
      sinks.n = 1;
    }
  }
  const auto* qh = static_cast<const __nv_bfloat16*>(q);
  const auto* kh = static_cast<const __nv_bfloat16*>(k);
  const auto* vh = static_cast<const __nv_bfloat16*>(v);
  launch_summary(qh, kh, vh, s, w, false, st);
  launch_kstats(s, w, st);
  launch_thresh(s, w, tau, false, st);
  cudaError_t re = launch_route_tc(&maps[5], s, w, sinks, d.status, st);
  if (re != cudaSuccess) return na_fail(SOL_ERR_LAUNCH, cudaGetErrorString(re));
  FwdParams p{};
  p.N = N;
  p.H = H;
  p.Nb = s.Nb;
  p.Nw = s.Nw;
  p.Na = s.Na;
  p.QT = s.QT;
  p.mask = w.mask;
  p.qt_begin = 0;
  p.qt_count = s.QT;
  p.row_lo = 0;
  p.row_hi = N;
  p.kv_splits = 1;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.status = d.status;
  cudaError_t e = launch_attn_fwd(maps, p, s.BH * s.QT, false, st);
  if (e != cudaSuccess) return na_fail(SOL_ERR_LAUNCH, cudaGetErrorString(e));
  e = cudaGetLastError();
  if (e != cudaSuccess) return na_fail(SOL_ERR_LAUNCH, cudaGetErrorString(e));
  return SOL_OK;
}

// Reads and clears the status word the allocation-free call's kernels write (a bounded wait that
// ran out, a misaligned shared-memory window).  Synchronises `stream` first; copies four bytes to a
// host variable and clears them with cudaMemset: nothing is allocated.
extern "C" int sol_attn_noalloc_get_device_status(void* stream) {
  set_last_error("");
  std::lock_guard<std::mutex> lock(g_na_mu);
  NoAllocDevice* d = nullptr;
  int rc = na_setup(&d);
  if (rc) return rc;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return na_fail(SOL_ERR_LAUNCH, "stream synchronisation failed");
  int h = 0;
  if (cudaMemcpy(&h, d->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess ||
      cudaMemset(d->status, 0, sizeof(int)) != cudaSuccess)
    return na_fail(SOL_ERR_LAUNCH, "status read failed");
  if (h == kDevTimeout) return na_fail(SOL_ERR_TIMEOUT, "a bounded wait inside a kernel ran out");
  if (h == kDevMisaligned) return na_fail(SOL_ERR_LAUNCH, "shared memory window misaligned; the kernel did not run");
  if (h == kDevBounds) return na_fail(SOL_ERR_LAUNCH, "a bounds check of the debug build failed (access skipped)");
  return SOL_OK;
}
