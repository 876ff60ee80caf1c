// Sol-Attn2 anchor tail statistics on the tensor cores.
//
// "Sol-Attn2: Sparse Attention with Complementary Approximation", Method, "Routing and
// complementary approximation": for a 32-token anchor with mean query qbar_a, over the tail groups
// g (the two key groups of every block outside E of the anchor's query block, non-empty ones only),
// w_ag = n_g exp(qbar_a . kbar_g / sqrt(d)), Z_a = sum_g w_ag, (mu_a, nu_a) = sum_g w_ag (kbar_g,
// vbar_g) / Z_a.
//
// This is an attention of the anchors over the groups with a per-group log-mass bias log n_g, a
// per-anchor mask (the exact blocks of its query block) and the 256-wide value [kbar_g | vbar_g].
// A CTA takes 128 anchors of one (b, h) (64 query blocks, M = 128 rows of tcgen05.mma) and streams
// the groups 128 at a time: S = Qa Kg^T (N = 128) into a double-buffered S in TMEM, a base-2 online
// softmax in one thread per anchor, P (BF16) written over the read S columns, and
// O += P [Kg | Vg] with N = 256 (the full-rate MMA shape) into a 256-column O in TMEM.
// Operands are BF16 (anchor means, group key / value means), accumulation FP32.
#include <cuda.h>
#include <cfloat>

#include "attn_fwd.cuh"
#include "common.cuh"
#include "ptx.cuh"

namespace sol {

namespace {

constexpr int kTailStages = 2;
constexpr uint32_t kHalf = 128 * 64 * 2;   // 128 rows x 64 BF16 columns, one 128-byte-swizzled half
constexpr uint32_t kColSt = 0, kColOt = 256;

struct __align__(1024) TailSmem {
  __nv_bfloat16 qa[2][128 * 64];                 // anchor means [d half][128 anchors x 64]
  __nv_bfloat16 g[kTailStages][4][128 * 64];     // [stage][kbar lo, kbar hi, vbar lo, vbar hi][128 groups x 64]
  uint64_t full[kTailStages], empty[kTailStages];
  uint64_t qfull, sfull[2], sfree[2], pready, pvdone, mmadone;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace

__global__ void __launch_bounds__(256, 1)
    tail_tc_kernel(const __grid_constant__ CUtensorMap tm_qa, const __grid_constant__ CUtensorMap tm_gk,
                   const __grid_constant__ CUtensorMap tm_gv, const Shape s, const Work w, int* status) {
  extern __shared__ __align__(1024) uint8_t tsm_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_u32(tsm_raw) & 1023u) {
    if (tid == 0) atomicExch(status, kDevMisaligned);
    return;
  }
  TailSmem& sm = *reinterpret_cast<TailSmem*>(tsm_raw);
  volatile int* abort = &sm.abort;
  const int bh = blockIdx.y;
  const int a0 = blockIdx.x * 128;
  const int ngroups = 2 * s.Nb;
  const int ntiles = (ngroups + 127) / 128;

  if (tid == 0) {
    for (int i = 0; i < kTailStages; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], 1);
    }
    mbar_init(&sm.qfull, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.sfull[i], 1);
      mbar_init(&sm.sfree[i], 1);
    }
    mbar_init(&sm.pready, 128);
    mbar_init(&sm.pvdone, 1);
    mbar_init(&sm.mmadone, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------------------------ loader
    if (lane == 0) {
      bool ok = true;
      mbar_arrive_expect_tx(&sm.qfull, 2 * kHalf);
      for (int dh = 0; dh < 2; ++dh) tma_load_3d(&sm.qa[dh][0], &tm_qa, &sm.qfull, 64 * dh, a0, bh);
      int t = 0;
      for (; t < ntiles && ok; ++t) {
        const int st = t % kTailStages;
        if (t >= kTailStages && !mbar_wait(&sm.empty[st], ((t / kTailStages) - 1) & 1, abort)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&sm.full[st], 4 * kHalf);
        for (int dh = 0; dh < 2; ++dh) {
          tma_load_3d(&sm.g[st][dh][0], &tm_gk, &sm.full[st], 64 * dh, 128 * t, bh);
          tma_load_3d(&sm.g[st][2 + dh][0], &tm_gv, &sm.full[st], 64 * dh, 128 * t, bh);
        }
      }
      if (!ok) atomicExch(status, kDevTimeout);
      for (int u = max(0, t - kTailStages); u < t; ++u)
        mbar_wait(&sm.full[u % kTailStages], (u / kTailStages) & 1, abort);
      mbar_wait(&sm.qfull, 0, abort);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(&sm.qfull, 0, abort);
      const uint32_t q_base = smem_u32(&sm.qa[0][0]);
      auto issue_pv = [&](int u) {
        if (!mbar_wait(&sm.pready, u & 1, abort)) return false;
        tc_fence_after();
        const int st = u % kTailStages;
        const uint32_t idesc = idesc_bf16(128, 256, false, true);
        const uint32_t v_base = smem_u32(&sm.g[st][0][0]);   // [kbar | vbar], four 64-channel atoms
        const uint32_t p_col = tmem + kColSt + 128 * (u & 1);
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bd = sdesc_sw128(v_base + kk * 2048, kHalf, 1024);
          umma_ts(tmem + kColOt, p_col + 8 * kk, bd, idesc, (u > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&sm.empty[st]);
        umma_commit(&sm.sfree[u & 1]);
        umma_commit(&sm.pvdone);
        return true;
      };
      for (int t = 0; t < ntiles && ok; ++t) {
        const int st = t % kTailStages;
        const int b = t & 1;
        if (!mbar_wait(&sm.full[st], (t / kTailStages) & 1, abort) ||
            (t >= 2 && !mbar_wait(&sm.sfree[b], ((t >> 1) - 1) & 1, abort))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(128, 128, false, false);
        const uint32_t k_base = smem_u32(&sm.g[st][0][0]);
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          umma_ss(tmem + kColSt + 128 * b, sdesc_sw128(q_base + off, 16, 1024), sdesc_sw128(k_base + off, 16, 1024),
                  idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sm.sfull[b]);
        if (t > 0 && !issue_pv(t - 1)) {
          ok = false;
          break;
        }
      }
      if (ok) ok = issue_pv(ntiles - 1);
      if (!ok) atomicExch(status, kDevTimeout);
      umma_commit(&sm.mmadone);
      mbar_wait(&sm.mmadone, 0, abort);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // -------------------------------------------------- softmax over the groups, one thread per anchor
    const int r = tid - 128;
    const int a = a0 + r;
    const bool a_valid = a < s.Na;
    const int qi = min(min(a, s.Na - 1) / 2, s.Nb - 1);
    const uint32_t* mrow = w.mask + ((size_t)bh * s.Nb + qi) * s.Nw;
    const float* lw2 = w.glog2n + (size_t)bh * tail_groups_padded(s);   // padded with -inf
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp - 4)) << 16);
    const float sc = kScale * kLog2e;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    int t = 0;
    for (; t < ntiles; ++t) {
      const int b = t & 1;
      if (!mbar_wait(&sm.sfull[b], (t >> 1) & 1, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t raw[128];
      const uint32_t s_addr = lane_addr + kColSt + 128 * b;
      tmem_ld32_at<0>(s_addr, raw);
      tmem_ld32_at<32>(s_addr + 32, raw);
      tmem_ld32_at<64>(s_addr + 64, raw);
      tmem_ld32_at<96>(s_addr + 96, raw);
      tmem_ld_wait();
      reg_fence(raw);
      // groups 128 t + c -> key block 64 t + c / 2; exact blocks of this anchor's query block and
      // empty groups are masked, the others get the bias log2 n_g
      const int wd = 2 * t;
      const uint32_t mw0 = wd < s.Nw ? mrow[wd] : 0xffffffffu;
      const uint32_t mw1 = wd + 1 < s.Nw ? mrow[wd + 1] : 0xffffffffu;
      float* x = reinterpret_cast<float*>(raw);
      float mp[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c4 = 0; c4 < 32; ++c4) {
        const float4 bias = *reinterpret_cast<const float4*>(lw2 + 128 * t + 4 * c4);
        const float bv[4] = {bias.x, bias.y, bias.z, bias.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = 4 * c4 + e;
          const int blk = c >> 1;   // 0 .. 63 within this tile
          const bool ex = ((blk < 32 ? mw0 : mw1) >> (blk & 31)) & 1u;
          x[c] = ex ? -INFINITY : fmaf(x[c], sc, bv[e]);
          mp[e] = fmaxf(mp[e], x[c]);
        }
      }
      const float mx = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3]));
      const float m_new = fmaxf(m_ref, mx);
      const bool upd = m_new > m_ref + 8.0f;
      const float m_use = upd ? m_new : m_ref;
      const float m_sub = m_use == -INFINITY ? 0.f : m_use;
      const float alpha = upd ? ex2f(m_ref - m_sub) : 1.f;
      float rs = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = ex2f(x[2 * c] - m_sub), p1 = ex2f(x[2 * c + 1] - m_sub);
        rs += p0 + p1;
        pk[c] = pack_bf16x2(p0, p1);
      }
      l = l * alpha + rs;
      if (t > 0 && !mbar_wait(&sm.pvdone, (t - 1) & 1, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      tmem_st32_at<0>(s_addr, pk);
      tmem_st32_at<32>(s_addr + 32, pk);
      const bool need = upd && t > 0 && m_ref != -INFINITY;
      if (__any_sync(0xffffffffu, need)) {
        const float f = need ? alpha : 1.f;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t o[64];
          tmem_ld32_at<0>(lane_addr + kColOt + 64 * q4, o);
          tmem_ld32_at<32>(lane_addr + kColOt + 64 * q4 + 32, o);
          tmem_ld_wait();
          reg_fence(o);
#pragma unroll
          for (int e = 0; e < 64; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
          tmem_st32_at<0>(lane_addr + kColOt + 64 * q4, o);
          tmem_st32_at<32>(lane_addr + kColOt + 64 * q4 + 32, o);
        }
      }
      m_ref = m_use;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&sm.pready);
    }
    if (ok && !mbar_wait(&sm.pvdone, (ntiles - 1) & 1, abort)) ok = false;
    if (!ok) atomicExch(status, kDevTimeout);
    tc_fence_after();
    if (__all_sync(0xffffffffu, ok)) {
      const bool has_tail = l > 0.f;
      const float inv = has_tail ? 1.f / l : 0.f;
      const size_t ab = (size_t)bh * s.Na + min(a, s.Na - 1);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t o[64];
        tmem_ld32_at<0>(lane_addr + kColOt + 64 * q4, o);
        tmem_ld32_at<32>(lane_addr + kColOt + 64 * q4 + 32, o);
        tmem_ld_wait();
        reg_fence(o);
        if (a_valid) {
          float* dst = (q4 < 2 ? w.tail_mu : w.tail_nu) + ab * kHeadDim + 64 * (q4 & 1);
#pragma unroll
          for (int e = 0; e < 64; e += 4)
            *reinterpret_cast<float4*>(dst + e) =
                make_float4(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv,
                            __uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
        }
      }
      if (a_valid) w.tail_logz[ab] = has_tail ? (m_ref + log2f(l)) * 0.69314718055994530942f : -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_tail_tc(const void* map_ptr, const Shape& s, const Work& w, int* status, cudaStream_t st) {
  const CUtensorMap* maps = static_cast<const CUtensorMap*>(map_ptr);
  const int smem = (int)sizeof(TailSmem);
  cudaError_t e = cudaFuncSetAttribute(tail_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  tail_tc_kernel<<<dim3((s.Na + 127) / 128, s.BH), 256, smem, st>>>(maps[0], maps[1], maps[2], s, w, status);
  return cudaGetLastError();
}

}  // namespace sol
