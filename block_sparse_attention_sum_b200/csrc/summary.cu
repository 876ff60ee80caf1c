// Block-summary, threshold-statistics and routing kernels of the Sol-Attn forward.
//
// Sol-Attn paper (arXiv 2607.24027): Eq. (3) pooled proxies, section 3.1 Eqs. (4)-(5) query-
// dependent threshold, section 3.2 on-the-fly thresholding; Sol-Attn README "Exact KV sink";
// stable-diffusion.cpp Sol-Attn documentation (adjacent blocks remain exact).
#include <cfloat>
#include <cmath>

#include "common.cuh"
#include "fp8.cuh"

namespace sol {

// -------------------------------------------------------------------------------------------------
// Block summaries.  One CTA per (key block j, batch b, head h).  Each 64-token block of one head is
// 64 rows of 256 contiguous bytes; 16 threads cover a row with 16-byte loads, 16 row groups cover
// the block, so every warp load instruction reads two full 256-byte rows.
// Outputs per (b, h, j): Qbar, Kbar (FP32 means over the valid tokens), BF16 copies of Kbar and
// of the value mean Vbar (surrogate MMA operands), and optionally the two 32-token anchor means of Q.
// -------------------------------------------------------------------------------------------------
// With kQuant (the FP8 path), the same pass also quantises Q and K per block (fp8.cuh,
// quant_block_rows) and folds the block's max |V| into the head's maximum.
template <bool kQuant>
__global__ void __launch_bounds__(256) summary_kernel(const __nv_bfloat16* __restrict__ q,
                                                      const __nv_bfloat16* __restrict__ k,
                                                      const __nv_bfloat16* __restrict__ v, Shape s, Work w,
                                                      int anchors, Fp8Work f8) {
  __shared__ float red[8][4][kHeadDim];
  __shared__ float qred[3 * 8];
  const int j = blockIdx.x, b = blockIdx.y / s.H, h = blockIdx.y % s.H;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c16 = tid & 15, rg = tid >> 4;
  const int t0 = j * kBlock;
  const int n = min(kBlock, s.N - t0);
  const int nlo = min(n, kAnchor), nhi = n - nlo;

  {
    float qlo[8], qhi[8], ks[8], vs[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) qlo[e] = qhi[e] = ks[e] = vs[e] = 0.f;
    uint4 rq[4], rk[4], rv[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int r = rg + 16 * m;
      if (r < n) {
        const size_t off = ((size_t)(b * (size_t)s.N + t0 + r) * s.H + h) * kHeadDim + 8 * c16;
        rq[m] = __ldg(reinterpret_cast<const uint4*>(q + off));
        rk[m] = __ldg(reinterpret_cast<const uint4*>(k + off));
        rv[m] = __ldg(reinterpret_cast<const uint4*>(v + off));
      } else {
        rq[m] = rk[m] = rv[m] = make_uint4(0, 0, 0, 0);
      }
    }
    // FP8 path: the block maxima of |Q|, |K|, |V| share the block synchronisation of the sums; Q and
    // K are quantised after the sums, once V's registers are free
    float mx[3];
    if (kQuant) {
      mx[0] = thread_absmax(rq);
      mx[1] = thread_absmax(rk);
      mx[2] = thread_absmax(rv);
      block_max_post(mx, qred);
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const __nv_bfloat162* pq = reinterpret_cast<const __nv_bfloat162*>(&rq[m]);
      const __nv_bfloat162* pk = reinterpret_cast<const __nv_bfloat162*>(&rk[m]);
      const __nv_bfloat162* pv = reinterpret_cast<const __nv_bfloat162*>(&rv[m]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 fq = __bfloat1622float2(pq[e]);
        float2 fk = __bfloat1622float2(pk[e]);
        float2 fv = __bfloat1622float2(pv[e]);
        if (m < 2) {
          qlo[2 * e] += fq.x;
          qlo[2 * e + 1] += fq.y;
        } else {
          qhi[2 * e] += fq.x;
          qhi[2 * e + 1] += fq.y;
        }
        ks[2 * e] += fk.x;
        ks[2 * e + 1] += fk.y;
        vs[2 * e] += fv.x;
        vs[2 * e + 1] += fv.y;
      }
    }
    // rows rg and rg ^ 1 live in lanes l and l ^ 16 of the same warp
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      qlo[e] += __shfl_xor_sync(0xffffffffu, qlo[e], 16);
      qhi[e] += __shfl_xor_sync(0xffffffffu, qhi[e], 16);
      ks[e] += __shfl_xor_sync(0xffffffffu, ks[e], 16);
      vs[e] += __shfl_xor_sync(0xffffffffu, vs[e], 16);
    }
    if (lane < 16) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        red[warp][0][8 * c16 + e] = qlo[e];
        red[warp][1][8 * c16 + e] = qhi[e];
        red[warp][2][8 * c16 + e] = ks[e];
        red[warp][3][8 * c16 + e] = vs[e];
      }
    }
    __syncthreads();
    if (tid < kHeadDim) {
      const int c = tid;
      float sqlo = 0.f, sqhi = 0.f, sk = 0.f, sv = 0.f;
#pragma unroll
      for (int ww = 0; ww < 8; ++ww) {
        sqlo += red[ww][0][c];
        sqhi += red[ww][1][c];
        sk += red[ww][2][c];
        sv += red[ww][3][c];
      }
      const size_t bh = (size_t)b * s.H + h;
      const size_t o = (bh * s.Nb + j) * kHeadDim + c;
      const float fn = (float)n;
      const float kb = sk / fn;
      const float qb = (sqlo + sqhi) / fn;
      w.qbar[o] = qb;
      w.kbar[o] = kb;
      const __nv_bfloat16 qh = __float2bfloat16_rn(qb), kh = __float2bfloat16_rn(kb);
      w.qbar_hi[o] = qh;
      w.qbar_lo[o] = __float2bfloat16_rn(qb - __bfloat162float(qh));
      w.kbar_h[o] = kh;
      w.kbar_lo[o] = __float2bfloat16_rn(kb - __bfloat162float(kh));
      w.vbar_h[o] = __float2bfloat16_rn(sv / fn);
      if (anchors) {
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
    }
    if (kQuant) {
      block_max_collect(mx, qred);
      const size_t bhj = ((size_t)b * s.H + h) * s.Nb + j;
      quant_block_rows(rq, mx[0], f8.q8, f8.sq + bhj, s.N, s.H, b, h, t0, n, tid);
      quant_block_rows(rk, mx[1], f8.k8, f8.sk + bhj, s.N, s.H, b, h, t0, n, tid);
      if (tid == 0) atomicMax(f8.vmax + (size_t)b * s.H + h, __float_as_uint(mx[2]));
    }
  }
}

// -------------------------------------------------------------------------------------------------
// Threshold statistics (Eq. (5)).  kmean = mean_j Kbar_j (FP64) and the centred covariance
// C = mean_j (Kbar_j - kmean)(Kbar_j - kmean)^T, so that sigma_i^2 = s^2 Qbar_i C Qbar_i^T equals
// Eq. (5)'s second moment minus mu_i^2 without its cancellation.  The Gram sum is split over
// kGramSplits ranges of key blocks (FP32 partial sums, 8 x 8 outputs per thread) and the partials
// are combined in FP64.
// -------------------------------------------------------------------------------------------------
constexpr int kGramSplits = 8;

// kmean: 8 row groups of 128 threads (thread = channel) sum every 8th key block with four
// independent FP64 accumulators each, then the groups combine in shared memory.
__global__ void __launch_bounds__(1024) kmean_kernel(Shape s, Work w) {
  __shared__ double part[8][kHeadDim];
  const int bh = blockIdx.x, c = threadIdx.x & (kHeadDim - 1), g = threadIdx.x >> 7;
  const float* kb = w.kbar + (size_t)bh * s.Nb * kHeadDim + c;
  double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
  int j = g;
  for (; j + 24 < s.Nb; j += 32) {
    a0 += (double)kb[(size_t)j * kHeadDim];
    a1 += (double)kb[(size_t)(j + 8) * kHeadDim];
    a2 += (double)kb[(size_t)(j + 16) * kHeadDim];
    a3 += (double)kb[(size_t)(j + 24) * kHeadDim];
  }
  for (; j < s.Nb; j += 8) a0 += (double)kb[(size_t)j * kHeadDim];
  part[g][c] = (a0 + a1) + (a2 + a3);
  __syncthreads();
  if (g == 0) {
    double acc = 0.0;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc += part[e][c];
    w.kmean[(size_t)bh * kHeadDim + c] = acc / s.Nb;
  }
}

__global__ void __launch_bounds__(256) kgram_kernel(Shape s, Work w, float* partial) {
  __shared__ __align__(16) float xs[32][kHeadDim];
  __shared__ float mk[kHeadDim];
  const int bh = blockIdx.y, split = blockIdx.x, tid = threadIdx.x;
  const int ti = tid >> 4, tj = tid & 15;
  const float* kb = w.kbar + (size_t)bh * s.Nb * kHeadDim;
  if (tid < kHeadDim) mk[tid] = (float)w.kmean[(size_t)bh * kHeadDim + tid];
  const int per = (s.Nb + kGramSplits - 1) / kGramSplits;
  const int j_lo = split * per, j_hi = min(s.Nb, j_lo + per);
  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[a][c] = 0.f;
  __syncthreads();
  for (int j0 = j_lo; j0 < j_hi; j0 += 32) {
    const int nj = min(32, j_hi - j0);
    for (int idx = tid; idx < 32 * kHeadDim; idx += 256) {
      const int jj = idx / kHeadDim, c = idx % kHeadDim;
      xs[jj][c] = jj < nj ? kb[(size_t)(j0 + jj) * kHeadDim + c] - mk[c] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int jj = 0; jj < 32; ++jj) {
      const float4 a0 = *reinterpret_cast<const float4*>(&xs[jj][8 * ti]);
      const float4 a1 = *reinterpret_cast<const float4*>(&xs[jj][8 * ti + 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&xs[jj][8 * tj]);
      const float4 b1 = *reinterpret_cast<const float4*>(&xs[jj][8 * tj + 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[a][c] = fmaf(av[a], bv[c], acc[a][c]);
    }
    __syncthreads();
  }
  float* out = partial + ((size_t)bh * kGramSplits + split) * kHeadDim * kHeadDim;
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    float4* row = reinterpret_cast<float4*>(out + (size_t)(8 * ti + a) * kHeadDim + 8 * tj);
    row[0] = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
    row[1] = make_float4(acc[a][4], acc[a][5], acc[a][6], acc[a][7]);
  }
}

__global__ void kgram_reduce_kernel(Shape s, Work w, const float* partial) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;   // entry of the 128 x 128 matrix
  if (e >= kHeadDim * kHeadDim) return;
  double acc = 0.0;
  for (int sp = 0; sp < kGramSplits; ++sp)
    acc += (double)partial[((size_t)bh * kGramSplits + sp) * kHeadDim * kHeadDim + e];
  w.kcov[(size_t)bh * kHeadDim * kHeadDim + e] = (float)(acc / s.Nb);
}

// -------------------------------------------------------------------------------------------------
// tau_i = mu_i + tau * sigma_i with mu_i = s Qbar_i . kmean and sigma_i^2 = s^2 Qbar_i C Qbar_i^T,
// stored as FP32, the precision the routing comparison is made in.  A CTA evaluates 64 rows:
// Y = Qbar C as a 64 x 128 x 128 product (4 rows x 8 columns per thread, FP32), then the row dot
// products Qbar_i . Y_i and Qbar_i . kmean.  Grid (ceil(Nb / 64), BH), 256 threads.
// -------------------------------------------------------------------------------------------------
constexpr int kThreshPad = 68;

__global__ void __launch_bounds__(256) thresh_kernel(Shape s, Work w, float tau, int diag) {
  extern __shared__ __align__(16) float tsm[];
  float* cov_s = tsm;                                // [128][128]
  float* qt = tsm + kHeadDim * kHeadDim;             // [128][68]  Qbar^T of the 64 rows
  __shared__ float part[64][17];
  __shared__ float mu_s[64];
  const int bh = blockIdx.y, i0 = blockIdx.x * 64, tid = threadIdx.x;
  const float* cov = w.kcov + (size_t)bh * kHeadDim * kHeadDim;
  const float* qb = w.qbar + (size_t)bh * s.Nb * kHeadDim;
  // all global loads of a thread are issued before the first shared-memory store, so they are in
  // flight together (16 x 16 bytes of the covariance, 8 x 16 bytes of the query-block means)
  {
    float4 cv[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) cv[e] = reinterpret_cast<const float4*>(cov)[tid + 256 * e];
    // lane = row (so the transposed shared-memory stores of a warp hit 32 consecutive words),
    // warp and e pick the four channels
    float4 qv[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int r = (tid & 31) + 32 * (e & 1), c4 = (tid >> 5) + 8 * (e >> 1);
      qv[e] = (i0 + r < s.Nb) ? reinterpret_cast<const float4*>(qb + (size_t)(i0 + r) * kHeadDim)[c4]
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) reinterpret_cast<float4*>(cov_s)[tid + 256 * e] = cv[e];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int r = (tid & 31) + 32 * (e & 1), c = 4 * ((tid >> 5) + 8 * (e >> 1));
      qt[(c + 0) * kThreshPad + r] = qv[e].x;
      qt[(c + 1) * kThreshPad + r] = qv[e].y;
      qt[(c + 2) * kThreshPad + r] = qv[e].z;
      qt[(c + 3) * kThreshPad + r] = qv[e].w;
    }
  }
  __syncthreads();
  if (tid < 64) {
    const double* mk = w.kmean + (size_t)bh * kHeadDim;
    double m = 0.0;
    for (int c = 0; c < kHeadDim; ++c) m += (double)qt[c * kThreshPad + tid] * mk[c];
    mu_s[tid] = (float)m;
  }
  if (diag) {
    // diagonal estimator: sigma_i^2 = s^2 sum_c Qbar_ic^2 C_cc
    if (tid < 64) {
      float q = 0.f;
      for (int c = 0; c < kHeadDim; ++c) {
        const float x = qt[c * kThreshPad + tid];
        q = fmaf(x * x, cov_s[c * kHeadDim + c], q);
      }
      part[tid][0] = q;
      for (int c = 1; c < 16; ++c) part[tid][c] = 0.f;
    }
  } else {
  const int ti = tid >> 4, tj = tid & 15;   // rows 4 ti .. 4 ti + 3, columns 8 tj .. 8 tj + 7
  float y[4][8];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) y[a][c] = 0.f;
#pragma unroll 4
  for (int d = 0; d < kHeadDim; ++d) {
    const float4 qa = *reinterpret_cast<const float4*>(&qt[d * kThreshPad + 4 * ti]);
    const float4 c0 = *reinterpret_cast<const float4*>(&cov_s[d * kHeadDim + 8 * tj]);
    const float4 c1 = *reinterpret_cast<const float4*>(&cov_s[d * kHeadDim + 8 * tj + 4]);
    const float av[4] = {qa.x, qa.y, qa.z, qa.w};
    const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 8; ++c) y[a][c] = fmaf(av[a], cv[c], y[a][c]);
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    float q = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) q = fmaf(qt[(8 * tj + c) * kThreshPad + 4 * ti + a], y[a][c], q);
    part[4 * ti + a][tj] = q;
  }
  }
  __syncthreads();
  if (tid < 64 && i0 + tid < s.Nb) {
    double quad = 0.0;
    for (int c = 0; c < 16; ++c) quad += (double)part[tid][c];
    const double sd = (double)kScale;
    const double m = sd * (double)mu_s[tid];
    const double var = fmax(sd * sd * quad, 0.0);
    w.thresh[(size_t)bh * s.Nb + i0 + tid] = (float)(m + (double)tau * sqrt(var));
  }
}

// Expand the bitmask into one byte per (query block, key block) pair (introspection only).
__global__ void expand_mask_kernel(Shape s, Work w, unsigned char* out) {
  const size_t total = (size_t)s.BH * s.Nb * s.Nb;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const size_t row = idx / s.Nb;
    const int j = (int)(idx % s.Nb);
    out[idx] = (w.mask[row * s.Nw + (j >> 5)] >> (j & 31)) & 1u;
  }
}

// Dense query rows: every key block exact for query blocks qb_lo + blockIdx.x.
__global__ void dense_mask_kernel(Shape s, Work w, int qb_lo) {
  const int i = qb_lo + blockIdx.x, bh = blockIdx.y;
  uint32_t* row = w.mask + ((size_t)bh * s.Nb + i) * s.Nw;
  for (int wd = threadIdx.x; wd < s.Nw; wd += blockDim.x) {
    const int nvalid = s.Nb - 32 * wd;
    row[wd] = nvalid >= 32 ? 0xffffffffu : ((1u << nvalid) - 1u);
  }
}

void launch_dense_mask(const Shape& s, const Work& w, int qb_lo, int qb_hi, cudaStream_t st) {
  dense_mask_kernel<<<dim3(qb_hi - qb_lo + 1, s.BH), 32, 0, st>>>(s, w, qb_lo);
}

void launch_summary(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, const Shape& s,
                    const Work& w, bool anchors, cudaStream_t st, const Fp8Work* f8) {
  if (f8)
    summary_kernel<true><<<dim3(s.Nb, s.BH), 256, 0, st>>>(q, k, v, s, w, anchors ? 1 : 0, *f8);
  else
    summary_kernel<false><<<dim3(s.Nb, s.BH), 256, 0, st>>>(q, k, v, s, w, anchors ? 1 : 0, Fp8Work{});
}

void launch_kstats(const Shape& s, const Work& w, cudaStream_t st) {
  kmean_kernel<<<s.BH, 8 * kHeadDim, 0, st>>>(s, w);
  kgram_kernel<<<dim3(kGramSplits, s.BH), 256, 0, st>>>(s, w, w.gram_partial);
  kgram_reduce_kernel<<<dim3(kHeadDim * kHeadDim / 256, s.BH), 256, 0, st>>>(s, w, w.gram_partial);
}

void launch_thresh(const Shape& s, const Work& w, float tau, bool diag, cudaStream_t st) {
  const int smem = (kHeadDim * kHeadDim + kHeadDim * kThreshPad) * sizeof(float);
  cudaFuncSetAttribute(thresh_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  thresh_kernel<<<dim3((s.Nb + 63) / 64, s.BH), 256, smem, st>>>(s, w, tau, diag ? 1 : 0);
}


void launch_expand_mask(const Shape& s, const Work& w, unsigned char* mask_out, cudaStream_t st) {
  expand_mask_kernel<<<1184, 256, 0, st>>>(s, w, mask_out);
}

}  // namespace sol
