// Routing on the tensor cores.
//
// Sol-Attn paper (arXiv 2607.24027), section 3.2, "Chunk-wise On-the-Fly Thresholding": block j is
// exact for query block i iff s_ij = s * Qbar_i . Kbar_j > tau_i, or |i - j| <= 1 (the adjacent
// blocks stay exact, stable-diffusion.cpp Sol-Attn documentation), or block j overlaps the sink
// (Sol-Attn README, "Exact KV sink").
//
// The proxies of one (b, h) form the product Qbar Kbar^T (Nb x 128 by 128 x Nb).  Each FP32 mean is
// split into two BF16 terms, x = x_hi + x_lo with x_hi = bf16(x) and x_lo = bf16(x - x_hi), and the
// product is taken as Qhi Khi^T + Qhi Klo^T + Qlo Khi^T with FP32 accumulation (the dropped
// Qlo Klo^T term and the rounding of the lo parts are about 2^-16 relative per term), so the
// decisions match an FP32 evaluation except for proxies within about 1e-4 of their threshold.
//
// A CTA takes 128 query blocks of one (b, h) (M = 128) and walks the key blocks 128 at a time
// (N = 128) through a 2-stage TMA ring; S goes to a double-buffered accumulator in TMEM and four
// epilogue warps (thread = query block) turn each 128-column slice into four bitmask words.  Only
// the bitmask, the per-row counts and the three routing statistics reach memory.
#include <cuda.h>

#include "common.cuh"
#include "ptx.cuh"

namespace sol {

namespace {

constexpr int kRtStages = 2;
constexpr uint32_t kRtHalf = 128 * 64 * 2;   // 128 rows x 64 BF16 channels, one swizzled half (16 KB)

struct __align__(1024) RouteSmem {
  __nv_bfloat16 q[2][2][128 * 64];               // [hi, lo][channel half][128 query blocks x 64]
  __nv_bfloat16 k[kRtStages][2][2][128 * 64];    // [stage][hi, lo][channel half][128 key blocks x 64]
  uint64_t full[kRtStages], empty[kRtStages], qfull, sfull[2], sfree[2], mmadone;
  uint32_t tmem_base;
  int abort;
};

}  // namespace

__global__ void __launch_bounds__(192, 1)
    route_tc_kernel(const __grid_constant__ CUtensorMap tm_qhi, const __grid_constant__ CUtensorMap tm_qlo,
                    const __grid_constant__ CUtensorMap tm_khi, const __grid_constant__ CUtensorMap tm_klo,
                    const Shape s, const Work w, const SinkSet sinks, int* status) {
  extern __shared__ __align__(1024) uint8_t rsm_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_u32(rsm_raw) & 1023u) {
    if (tid == 0) atomicExch(status, kDevMisaligned);
    return;
  }
  RouteSmem& sm = *reinterpret_cast<RouteSmem*>(rsm_raw);
  volatile int* abort = &sm.abort;
  const int bh = blockIdx.y;
  const int i0 = blockIdx.x * 128;
  const int nchunks = (s.Nb + 127) / 128;

  if (tid == 0) {
    for (int i = 0; i < kRtStages; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], 1);
    }
    mbar_init(&sm.qfull, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.sfull[i], 1);
      mbar_init(&sm.sfree[i], 128);
    }
    mbar_init(&sm.mmadone, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------------------- TMA loads
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(&sm.qfull, 4 * kRtHalf);
      for (int dh = 0; dh < 2; ++dh) {
        tma_load_3d(&sm.q[0][dh][0], &tm_qhi, &sm.qfull, 64 * dh, i0, bh);
        tma_load_3d(&sm.q[1][dh][0], &tm_qlo, &sm.qfull, 64 * dh, i0, bh);
      }
      int c = 0;
      for (; c < nchunks; ++c) {
        const int st = c % kRtStages;
        if (c >= kRtStages && !mbar_wait(&sm.empty[st], ((c / kRtStages) - 1) & 1, abort)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&sm.full[st], 4 * kRtHalf);
        for (int dh = 0; dh < 2; ++dh) {
          tma_load_3d(&sm.k[st][0][dh][0], &tm_khi, &sm.full[st], 64 * dh, 128 * c, bh);
          tma_load_3d(&sm.k[st][1][dh][0], &tm_klo, &sm.full[st], 64 * dh, 128 * c, bh);
        }
      }
      if (!ok) atomicExch(status, kDevTimeout);
      // never leave the CTA with bulk copies in flight
      for (int u = max(0, c - kRtStages); u < c; ++u) mbar_wait(&sm.full[u % kRtStages], (u / kRtStages) & 1, abort);
      mbar_wait(&sm.qfull, 0, abort);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(&sm.qfull, 0, abort);
      const uint32_t idesc = idesc_bf16(128, 128, false, false);
      const uint32_t qh = smem_u32(&sm.q[0][0][0]), ql = smem_u32(&sm.q[1][0][0]);
      for (int c = 0; c < nchunks && ok; ++c) {
        const int st = c % kRtStages;
        const int b = c & 1;
        if (!mbar_wait(&sm.full[st], (c / kRtStages) & 1, abort) ||
            (c >= 2 && !mbar_wait(&sm.sfree[b], ((c >> 1) - 1) & 1, abort))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kh = smem_u32(&sm.k[st][0][0][0]), kl = smem_u32(&sm.k[st][1][0][0]);
        // the two cross terms first, then the leading term
        const uint32_t a_op[3] = {qh, ql, qh}, b_op[3] = {kl, kh, kh};
        for (int term = 0; term < 3; ++term) {
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kRtHalf + (kk & 3) * 32;
            umma_ss(tmem + 128 * b, sdesc_sw128(a_op[term] + off, 16, 1024), sdesc_sw128(b_op[term] + off, 16, 1024),
                    idesc, (term > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&sm.sfull[b]);
        umma_commit(&sm.empty[st]);
      }
      if (!ok) atomicExch(status, kDevTimeout);
      umma_commit(&sm.mmadone);
      mbar_wait(&sm.mmadone, 0, abort);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------- decisions: one thread per query block (TMEM lane)
    const int q4 = warp & 3;   // warps 2..5 -> TMEM lane quarters 2, 3, 0, 1
    const int r = 32 * q4 + lane;
    const int i = i0 + r;
    const bool row_in = i < s.Nb;
    const float th = row_in ? w.thresh[(size_t)bh * s.Nb + i] : 0.f;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * q4) << 16);
    uint32_t* mrow = w.mask + ((size_t)bh * s.Nb + min(i, s.Nb - 1)) * s.Nw;
    int count = 0;
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
      const int b = c & 1;
      if (!mbar_wait(&sm.sfull[b], (c >> 1) & 1, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[128];
      tmem_ld32_at<0>(lane_addr + 128 * b, v);
      tmem_ld32_at<32>(lane_addr + 128 * b + 32, v);
      tmem_ld32_at<64>(lane_addr + 128 * b + 64, v);
      tmem_ld32_at<96>(lane_addr + 128 * b + 96, v);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&sm.sfree[b]);   // the accumulator may be overwritten (values are in registers)
      uint32_t words[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t bits = 0;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float shat = __uint_as_float(v[32 * g + e]) * kScale;
          bits |= (shat > th ? 1u : 0u) << e;
        }
        const int jb = 128 * c + 32 * g;   // first key block of this word
        // forced blocks: adjacency and the sink; nothing beyond the last block
        for (int j = max(i - 1, jb); j <= min(i + 1, jb + 31); ++j) bits |= 1u << (j - jb);
        for (int e = 0; e < sinks.n; ++e) {
          const int lo = max(sinks.b0[e], jb), hi = min(sinks.b1[e], jb + 31);
          for (int j = lo; j <= hi; ++j) bits |= 1u << (j - jb);
        }
        const int nvalid = s.Nb - jb;
        if (nvalid < 32) bits &= nvalid > 0 ? ((1u << nvalid) - 1u) : 0u;
        words[g] = bits;
      }
      if (row_in) {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int wd = 4 * c + g;
          if (wd < s.Nw) {
            mrow[wd] = words[g];
            count += __popc(words[g]);
          }
        }
      }
    }
    if (!ok) atomicExch(status, kDevTimeout);
    if (ok && row_in) {
      w.rowcount[(size_t)bh * s.Nb + i] = count;
      atomicAdd(&w.stats[0], (unsigned long long)count);
      atomicMin(&w.stats[1], (unsigned long long)count);
      atomicMax(&w.stats[2], (unsigned long long)count);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

cudaError_t launch_route_tc(const void* map_ptr, const Shape& s, const Work& w, const SinkSet& sinks, int* status,
                            cudaStream_t st) {
  const CUtensorMap* maps = static_cast<const CUtensorMap*>(map_ptr);
  const int smem = (int)sizeof(RouteSmem);
  cudaError_t e = cudaFuncSetAttribute(route_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  route_tc_kernel<<<dim3((s.Nb + 127) / 128, s.BH), 192, smem, st>>>(maps[0], maps[1], maps[2], maps[3], s, w, sinks,
                                                                      status);
  return cudaGetLastError();
}

}  // namespace sol
