// Sol-Attn2 complementary tail: the key groups.
//
// "Sol-Attn2: Sparse Attention with Complementary Approximation", Method, "Routing and
// complementary approximation": each unselected key block is split into two content groups by its
// keys' projection on the mean-query direction.  The direction is the mean of all queries of the
// (batch, head), so the groups do not depend on the query and are built once here, for every key
// block, in the same pass over K and V that computes the block means: a query pass (query and
// anchor means), the direction, then the key / value pass.  The per-anchor tail statistics over
// the groups are computed on the tensor cores (sol2_tail_tc.cu).
#include <cfloat>
#include <cmath>

#include "common.cuh"
#include "fp8.cuh"

namespace sol {

// u = mean of all queries of a (b, h) = sum_j n_j Qbar_j / N, accumulated in FP64.  Also marks the
// padding groups 2 Nb .. Gp - 1 of the log-size row as empty.
// Eight row groups of 128 threads (thread = channel) sum every eighth block, then combine.
__global__ void __launch_bounds__(1024) qdir_kernel(Shape s, Work w) {
  __shared__ double part[8][kHeadDim];
  const int bh = blockIdx.x, c = threadIdx.x & (kHeadDim - 1), g = threadIdx.x >> 7;
  const int gp = tail_groups_padded(s);
  if (g == 0 && 2 * s.Nb + c < gp) w.glog2n[(size_t)bh * gp + 2 * s.Nb + c] = -INFINITY;
  const float* qb = w.qbar + (size_t)bh * s.Nb * kHeadDim + c;
  double a0 = 0.0, a1 = 0.0;
  int j = g;
  for (; j + 8 < s.Nb; j += 16) {
    a0 += (double)min(kBlock, s.N - j * kBlock) * (double)qb[(size_t)j * kHeadDim];
    a1 += (double)min(kBlock, s.N - (j + 8) * kBlock) * (double)qb[(size_t)(j + 8) * kHeadDim];
  }
  for (; j < s.Nb; j += 8) a0 += (double)min(kBlock, s.N - j * kBlock) * (double)qb[(size_t)j * kHeadDim];
  part[g][c] = a0 + a1;
  __syncthreads();
  if (g == 0) {
    double acc = 0.0;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc += part[e][c];
    w.qdir[(size_t)bh * kHeadDim + c] = (float)(acc / s.N);
  }
}

// Query pass of the Sol-Attn2 summaries: Qbar (FP32 and the BF16 hi / lo split of the routing
// product) and the two 32-token anchor means of every block.  One CTA per (query block j, b, h)
// with summary_kernel's thread mapping and summation order, so Qbar is bit-identical to the
// Sol-Attn path's.
template <bool kQuant>
__global__ void __launch_bounds__(256) summary_q_kernel(const __nv_bfloat16* __restrict__ q, Shape s, Work w,
                                                        Fp8Work f8) {
  __shared__ float red[8][2][kHeadDim];
  __shared__ float qred[8];
  const int j = blockIdx.x, b = blockIdx.y / s.H, h = blockIdx.y % s.H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c16 = tid & 15, rg = tid >> 4;
  const int t0 = j * kBlock;
  const int n = min(kBlock, s.N - t0);
  const int nlo = min(n, kAnchor), nhi = n - nlo;
  float qlo[8], qhi[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) qlo[e] = qhi[e] = 0.f;
  uint4 rq[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int r = rg + 16 * m;
    rq[m] = r < n ? __ldg(reinterpret_cast<const uint4*>(q + ((size_t)(b * (size_t)s.N + t0 + r) * s.H + h) * kHeadDim +
                                                        8 * c16))
                  : make_uint4(0, 0, 0, 0);
  }
  // the FP8 path: Q codes and the block's scale in the same pass (the maximum shares the block
  // synchronisation of the sums)
  float mq[1];
  if (kQuant) {
    mq[0] = thread_absmax(rq);
    block_max_post(mq, qred);
  }
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const __nv_bfloat162* pq = reinterpret_cast<const __nv_bfloat162*>(&rq[m]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fq = __bfloat1622float2(pq[e]);
      if (m < 2) {
        qlo[2 * e] += fq.x;
        qlo[2 * e + 1] += fq.y;
      } else {
        qhi[2 * e] += fq.x;
        qhi[2 * e + 1] += fq.y;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    qlo[e] += __shfl_xor_sync(0xffffffffu, qlo[e], 16);
    qhi[e] += __shfl_xor_sync(0xffffffffu, qhi[e], 16);
  }
  if (lane < 16) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      red[warp][0][8 * c16 + e] = qlo[e];
      red[warp][1][8 * c16 + e] = qhi[e];
    }
  }
  __syncthreads();
  if (tid < kHeadDim) {
    const int c = tid;
    float sqlo = 0.f, sqhi = 0.f;
#pragma unroll
    for (int ww = 0; ww < 8; ++ww) {
      sqlo += red[ww][0][c];
      sqhi += red[ww][1][c];
    }
    const size_t bh = (size_t)b * s.H + h;
    const size_t o = (bh * s.Nb + j) * kHeadDim + c;
    const float qb = (sqlo + sqhi) / (float)n;
    w.qbar[o] = qb;
    const __nv_bfloat16 qh = __float2bfloat16_rn(qb);
    w.qbar_hi[o] = qh;
    w.qbar_lo[o] = __float2bfloat16_rn(qb - __bfloat162float(qh));
    const size_t a0 = (bh * s.Na + 2 * (size_t)j) * kHeadDim + c;
    const float alo = sqlo / (float)nlo;
    w.qanchor[a0] = alo;
    w.qanchor_h[a0] = __float2bfloat16_rn(alo);
    if (nhi > 0) {
      const float ahi = sqhi / (float)nhi;
      w.qanchor[a0 + kHeadDim] = ahi;
      w.qanchor_h[a0 + kHeadDim] = __float2bfloat16_rn(ahi);
    }
  }
  if (kQuant) {
    block_max_collect(mq, qred);
    quant_block_rows(rq, mq[0], f8.q8, f8.sq + ((size_t)b * s.H + h) * s.Nb + j, s.N, s.H, b, h, t0, n, tid);
  }
}

// Key / value pass of the Sol-Attn2 summaries, after the mean query u is known: Kbar (FP32 and the
// BF16 hi / lo split of the routing product; summary_kernel's summation order, so bit-identical)
// and the block's two key groups: group 1 = keys with k.u > Kbar_j.u, group 0 = the rest (FP32
// decision), their sizes, key means and value means.  K and V are read once, kept in registers
// between the block-mean reduction and the group split.  One CTA per (key block j, b, h): 16
// threads cover a 256-byte row with 16-byte loads, 16 row groups cover the block.
template <bool kQuant>
__global__ void __launch_bounds__(256) summary_kv_groups_kernel(const __nv_bfloat16* __restrict__ k,
                                                                const __nv_bfloat16* __restrict__ v, Shape s, Work w,
                                                                Fp8Work f8) {
  __shared__ float red[8][4][kHeadDim];
  __shared__ float qred[2 * 8];
  __shared__ float kbar_s[kHeadDim];
  __shared__ int n1_s;
  const int j = blockIdx.x, bh = blockIdx.y, b = bh / s.H, h = bh % s.H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c16 = tid & 15, rg = tid >> 4;
  const int t0 = j * kBlock;
  const int n = min(kBlock, s.N - t0);
  if (tid == 0) n1_s = 0;
  uint4 rk[4], rv[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int r = rg + 16 * m;
    if (r < n) {
      const size_t off = ((size_t)(b * (size_t)s.N + t0 + r) * s.H + h) * kHeadDim + 8 * c16;
      rk[m] = __ldg(reinterpret_cast<const uint4*>(k + off));
      rv[m] = __ldg(reinterpret_cast<const uint4*>(v + off));
    } else {
      rk[m] = rv[m] = make_uint4(0, 0, 0, 0);
    }
  }
  // the FP8 path: K codes and the block's scale, max |V| into the head's maximum; the maxima share
  // the block synchronisation of the key mean
  float mx[2];
  if (kQuant) {
    mx[0] = thread_absmax(rk);
    mx[1] = thread_absmax(rv);
    block_max_post(mx, qred);
  }
  // ---- block mean of the keys
  {
    float ks[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) ks[e] = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const __nv_bfloat162* pk = reinterpret_cast<const __nv_bfloat162*>(&rk[m]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fk = __bfloat1622float2(pk[e]);
        ks[2 * e] += fk.x;
        ks[2 * e + 1] += fk.y;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) ks[e] += __shfl_xor_sync(0xffffffffu, ks[e], 16);
    if (lane < 16) {
#pragma unroll
      for (int e = 0; e < 8; ++e) red[warp][0][8 * c16 + e] = ks[e];
    }
    __syncthreads();
    if (kQuant) {
      block_max_collect(mx, qred);
      quant_block_rows(rk, mx[0], f8.k8, f8.sk + (size_t)bh * s.Nb + j, s.N, s.H, b, h, t0, n, tid);
      if (tid == 0) atomicMax(f8.vmax + bh, __float_as_uint(mx[1]));
    }
    if (tid < kHeadDim) {
      const int c = tid;
      float sk = 0.f;
#pragma unroll
      for (int ww = 0; ww < 8; ++ww) sk += red[ww][0][c];
      const size_t o = ((size_t)bh * s.Nb + j) * kHeadDim + c;
      const float kb = sk / (float)n;
      w.kbar[o] = kb;
      const __nv_bfloat16 kh = __float2bfloat16_rn(kb);
      w.kbar_h[o] = kh;
      w.kbar_lo[o] = __float2bfloat16_rn(kb - __bfloat162float(kh));
      kbar_s[c] = kb;
    }
    __syncthreads();
  }
  // ---- the two groups: the cut Kbar_j . u, reduced over the 16 lanes of a row group
  const float* u = w.qdir + (size_t)bh * kHeadDim + 8 * c16;
  float uu[8];
  float cut = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    uu[e] = u[e];
    cut = fmaf(kbar_s[8 * c16 + e], uu[e], cut);
  }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) cut += __shfl_xor_sync(0xffffffffu, cut, o);
  float k0[8], k1[8], v0[8], v1[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) k0[e] = k1[e] = v0[e] = v1[e] = 0.f;
  int n1 = 0;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const bool valid = rg + 16 * m < n;   // uniform across the 16 lanes of the row
    float fk[8], fv[8];
    const __nv_bfloat162* pk = reinterpret_cast<const __nv_bfloat162*>(&rk[m]);
    const __nv_bfloat162* pv = reinterpret_cast<const __nv_bfloat162*>(&rv[m]);
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
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) proj += __shfl_xor_sync(0xffffffffu, proj, o);
    const bool upper = valid && proj > cut;
    n1 += upper ? 1 : 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      k1[e] += upper ? fk[e] : 0.f;
      v1[e] += upper ? fv[e] : 0.f;
      k0[e] += upper ? 0.f : fk[e];
      v0[e] += upper ? 0.f : fv[e];
    }
  }
  // rows rg and rg + 1 of a warp live in lanes l and l ^ 16
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
    const size_t g0 = (((size_t)bh * s.Nb + j) * 2) * kHeadDim + c;
    w.gk_h[g0] = __float2bfloat16_rn(cnt0 ? a0 / (float)cnt0 : 0.f);
    w.gv_h[g0] = __float2bfloat16_rn(cnt0 ? b0 / (float)cnt0 : 0.f);
    w.gk_h[g0 + kHeadDim] = __float2bfloat16_rn(cnt1 ? a1 / (float)cnt1 : 0.f);
    w.gv_h[g0 + kHeadDim] = __float2bfloat16_rn(cnt1 ? b1 / (float)cnt1 : 0.f);
    if (c < 2) {
      const int cnt = c == 0 ? cnt0 : cnt1;
      w.glog2n[(size_t)bh * tail_groups_padded(s) + 2 * j + c] = cnt > 0 ? log2f((float)cnt) : -INFINITY;
    }
  }
}

void launch_sol2_summaries(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, const Shape& s,
                           const Work& w, cudaStream_t st, const Fp8Work* f8) {
  if (f8)
    summary_q_kernel<true><<<dim3(s.Nb, s.BH), 256, 0, st>>>(q, s, w, *f8);
  else
    summary_q_kernel<false><<<dim3(s.Nb, s.BH), 256, 0, st>>>(q, s, w, Fp8Work{});
  qdir_kernel<<<s.BH, 8 * kHeadDim, 0, st>>>(s, w);
  if (f8)
    summary_kv_groups_kernel<true><<<dim3(s.Nb, s.BH), 256, 0, st>>>(k, v, s, w, *f8);
  else
    summary_kv_groups_kernel<false><<<dim3(s.Nb, s.BH), 256, 0, st>>>(k, v, s, w, Fp8Work{});
}

}  // namespace sol
