// Sol-Attn2 complementary tail: key groups and per-anchor tail statistics.
//
// "Sol-Attn2: Sparse Attention with Complementary Approximation", Method, "Routing and
// complementary approximation": each unselected key block is split into two content groups by its
// keys' projection on the mean-query direction; for a 32-token anchor with mean query qbar_a,
// w_ag = n_g exp(qbar_a . kbar_g / sqrt(d)), Z_a = sum_g w_ag, (mu_a, nu_a) = sum_g w_ag (kbar_g,
// vbar_g) / Z_a over the tail groups (the groups of the blocks outside E of the anchor's query block).
// The direction is the mean of all queries of the (batch, head), so the groups do not depend on the
// query and are built once here.
#include <cfloat>
#include <cmath>

#include "common.cuh"

namespace sol {

// u = mean of all queries of a (b, h) = sum_j n_j Qbar_j / N, accumulated in FP64.
__global__ void qdir_kernel(Shape s, Work w) {
  const int bh = blockIdx.x, c = threadIdx.x;
  const float* qb = w.qbar + (size_t)bh * s.Nb * kHeadDim;
  double acc = 0.0;
  for (int j = 0; j < s.Nb; ++j) {
    const int n = min(kBlock, s.N - j * kBlock);
    acc += (double)n * (double)qb[(size_t)j * kHeadDim + c];
  }
  w.qdir[(size_t)bh * kHeadDim + c] = (float)(acc / s.N);
}

// Two groups per key block: group 1 = keys with k.u > Kbar_j.u, group 0 = the rest (FP32 decision).
// Same access pattern as the block-summary kernel: one CTA per (key block, batch), heads in turn.
__global__ void __launch_bounds__(256) groups_kernel(const __nv_bfloat16* __restrict__ k,
                                                     const __nv_bfloat16* __restrict__ v, Shape s, Work w) {
  __shared__ float red[8][4][kHeadDim];
  __shared__ float cut_s;
  __shared__ int n1_s;
  const int j = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c16 = tid & 15, rg = tid >> 4;
  const int t0 = j * kBlock;
  const int n = min(kBlock, s.N - t0);
  for (int h = 0; h < s.H; ++h) {
    const size_t bh = (size_t)b * s.H + h;
    const float* u = w.qdir + bh * kHeadDim;
    if (warp == 0) {
      const float* kb = w.kbar + (bh * s.Nb + j) * kHeadDim;
      float acc = 0.f;
      for (int c = lane; c < kHeadDim; c += 32) acc = fmaf(kb[c], u[c], acc);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) {
        cut_s = acc;
        n1_s = 0;
      }
    }
    float uu[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) uu[e] = u[8 * c16 + e];
    __syncthreads();
    const float cut = cut_s;
    float k0[8], k1[8], v0[8], v1[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) k0[e] = k1[e] = v0[e] = v1[e] = 0.f;
    int n1 = 0;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int r = rg + 16 * m;
      const bool valid = r < n;   // uniform across the 16 lanes of the row
      uint4 rk = make_uint4(0, 0, 0, 0), rv = make_uint4(0, 0, 0, 0);
      if (valid) {
        const size_t off = ((size_t)(b * (size_t)s.N + t0 + r) * s.H + h) * kHeadDim + 8 * c16;
        rk = __ldg(reinterpret_cast<const uint4*>(k + off));
        rv = __ldg(reinterpret_cast<const uint4*>(v + off));
      }
      float fk[8], fv[8];
      const __nv_bfloat162* pk = reinterpret_cast<const __nv_bfloat162*>(&rk);
      const __nv_bfloat162* pv = reinterpret_cast<const __nv_bfloat162*>(&rv);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 a = __bfloat1622float2(pk[e]);
        const float2 c = __bfloat1622float2(pv[e]);
        fk[2 * e] = a.x;
        fk[2 * e + 1] = a.y;
        fv[2 * e] = c.x;
        fv[2 * e + 1] = c.y;
      }
      float proj = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) proj = fmaf(fk[e], uu[e], proj);
      // the 16 lanes of one row are lanes (lane & 16) .. (lane & 16) + 15
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) proj += __shfl_xor_sync(0xffffffffu, proj, o);
      const bool upper = valid && proj > cut;
      if (valid && c16 == 0 && upper) ++n1;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (upper) {
          k1[e] += fk[e];
          v1[e] += fv[e];
        } else {
          k0[e] += fk[e];
          v0[e] += fv[e];
        }
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      k0[e] += __shfl_xor_sync(0xffffffffu, k0[e], 16);
      k1[e] += __shfl_xor_sync(0xffffffffu, k1[e], 16);
      v0[e] += __shfl_xor_sync(0xffffffffu, v0[e], 16);
      v1[e] += __shfl_xor_sync(0xffffffffu, v1[e], 16);
    }
    if (c16 == 0 && n1) atomicAdd(&n1_s, n1);
    if (lane < 16) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        red[warp][0][8 * c16 + e] = k0[e];
        red[warp][1][8 * c16 + e] = k1[e];
        red[warp][2][8 * c16 + e] = v0[e];
        red[warp][3][8 * c16 + e] = v1[e];
      }
    }
    __syncthreads();
    if (tid < kHeadDim) {
      const int c = tid;
      float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
      for (int ww = 0; ww < 8; ++ww) {
        a0 += red[ww][0][c];
        a1 += red[ww][1][c];
        b0 += red[ww][2][c];
        b1 += red[ww][3][c];
      }
      const int cnt1 = n1_s, cnt0 = n - cnt1;
      const size_t g0 = ((bh * s.Nb + j) * 2) * kHeadDim + c;
      w.gk[g0] = cnt0 ? a0 / (float)cnt0 : 0.f;
      w.gv[g0] = cnt0 ? b0 / (float)cnt0 : 0.f;
      w.gk[g0 + kHeadDim] = cnt1 ? a1 / (float)cnt1 : 0.f;
      w.gv[g0 + kHeadDim] = cnt1 ? b1 / (float)cnt1 : 0.f;
      if (c == 0) {
        w.gcount[(bh * s.Nb + j) * 2] = cnt0;
        w.gcount[(bh * s.Nb + j) * 2 + 1] = cnt1;
      }
    }
    __syncthreads();
  }
}

// Per-anchor tail statistics.  CTA = (64 anchors, one (b, h)); thread = (anchor, channel slice),
// slice s owns channels 4e + s.  Groups stream through shared memory 32 at a time; each anchor keeps
// an online log-sum-exp (max, Z) and the weighted key / value sums of its slice.
constexpr int kTailAnchors = 64;
constexpr int kTailGroups = 32;

__global__ void __launch_bounds__(256, 1) anchor_tail_kernel(Shape s, Work w) {
  __shared__ float gk_s[kTailGroups][kHeadDim];
  __shared__ float gv_s[kTailGroups][kHeadDim];
  __shared__ float lw_s[kTailGroups];   // ln n_g, or -inf for an empty group
  const int bh = blockIdx.y, tid = threadIdx.x;
  const int al = tid >> 2, sl = tid & 3;
  const int a = blockIdx.x * kTailAnchors + al;
  const bool a_valid = a < s.Na;
  const int qi = min(a, s.Na - 1) / 2;   // query block of the anchor
  const uint32_t* mrow = w.mask + ((size_t)bh * s.Nb + min(qi, s.Nb - 1)) * s.Nw;
  float qa[32];
  const float* qap = w.qanchor + ((size_t)bh * s.Na + min(a, s.Na - 1)) * kHeadDim;
#pragma unroll
  for (int e = 0; e < 32; ++e) qa[e] = qap[4 * e + sl];
  float acck[32], accv[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) acck[e] = accv[e] = 0.f;
  float m = -INFINITY, Z = 0.f;
  const int ngroups = 2 * s.Nb;
  for (int g0 = 0; g0 < ngroups; g0 += kTailGroups) {
    __syncthreads();
    for (int idx = tid; idx < kTailGroups * kHeadDim; idx += 256) {
      const int gg = idx / kHeadDim, c = idx % kHeadDim;
      const int g = g0 + gg;
      const bool in = g < ngroups;
      gk_s[gg][c] = in ? w.gk[((size_t)bh * ngroups + g) * kHeadDim + c] : 0.f;
      gv_s[gg][c] = in ? w.gv[((size_t)bh * ngroups + g) * kHeadDim + c] : 0.f;
    }
    if (tid < kTailGroups) {
      const int g = g0 + tid;
      const int cnt = g < ngroups ? w.gcount[(size_t)bh * ngroups + g] : 0;
      lw_s[tid] = cnt > 0 ? logf((float)cnt) : -INFINITY;
    }
    __syncthreads();
    // the 32 groups are 16 key blocks j0 .. j0 + 15 with j0 = g0 / 2
    const int j0 = g0 >> 1;
    const uint32_t word = mrow[j0 >> 5];
    const uint32_t ex16 = (word >> (j0 & 31)) & 0xffffu;   // j0 is a multiple of 16
#pragma unroll 1
    for (int g8 = 0; g8 < kTailGroups; g8 += 8) {
      float logit[8];
#pragma unroll
      for (int gg = 0; gg < 8; ++gg) {
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) part = fmaf(qa[e], gk_s[g8 + gg][4 * e + sl], part);
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);
        const bool exact = (ex16 >> ((g8 + gg) >> 1)) & 1u;
        logit[gg] = exact ? -INFINITY : fmaf(part, kScale, lw_s[g8 + gg]);
      }
      float mx = m;
#pragma unroll
      for (int gg = 0; gg < 8; ++gg) mx = fmaxf(mx, logit[gg]);
      if (mx == -INFINITY) continue;
      if (mx > m) {   // new running max: rescale the accumulators
        const float alpha = __expf(m - mx);
        Z *= alpha;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          acck[e] *= alpha;
          accv[e] *= alpha;
        }
        m = mx;
      }
#pragma unroll
      for (int gg = 0; gg < 8; ++gg) {
        const float wgt = __expf(logit[gg] - m);
        Z += wgt;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          acck[e] = fmaf(wgt, gk_s[g8 + gg][4 * e + sl], acck[e]);
          accv[e] = fmaf(wgt, gv_s[g8 + gg][4 * e + sl], accv[e]);
        }
      }
    }
  }
  if (!a_valid) return;
  const size_t ab = (size_t)bh * s.Na + a;
  if (Z > 0.f) {
    const float inv = 1.f / Z;
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      w.tail_mu[ab * kHeadDim + 4 * e + sl] = acck[e] * inv;
      w.tail_nu[ab * kHeadDim + 4 * e + sl] = accv[e] * inv;
    }
    if (sl == 0) w.tail_logz[ab] = m + logf(Z);
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      w.tail_mu[ab * kHeadDim + 4 * e + sl] = 0.f;
      w.tail_nu[ab * kHeadDim + 4 * e + sl] = 0.f;
    }
    if (sl == 0) w.tail_logz[ab] = -INFINITY;
  }
}

void launch_groups(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, const Shape& s,
                   const Work& w, cudaStream_t st) {
  (void)q;
  qdir_kernel<<<s.BH, kHeadDim, 0, st>>>(s, w);
  groups_kernel<<<dim3(s.Nb, s.B), 256, 0, st>>>(k, v, s, w);
}

void launch_anchor_tail(const Shape& s, const Work& w, cudaStream_t st) {
  anchor_tail_kernel<<<dim3((s.Na + kTailAnchors - 1) / kTailAnchors, s.BH), 256, 0, st>>>(s, w);
}

}  // namespace sol
