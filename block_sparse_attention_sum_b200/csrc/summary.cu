// Block-summary, threshold-statistics and routing kernels of the Sol-Attn forward.
//
// Sol-Attn paper (arXiv 2607.24027): Eq. (3) pooled proxies, section 3.1 Eqs. (4)-(5) query-
// dependent threshold, section 3.2 on-the-fly thresholding; Sol-Attn README "Exact KV sink";
// stable-diffusion.cpp Sol-Attn documentation (adjacent blocks remain exact).
#include <cfloat>
#include <cmath>

#include "common.cuh"

namespace sol {

// -------------------------------------------------------------------------------------------------
// Block summaries.  One CTA per (key block j, batch b); it walks the heads.  Each 64-token block of
// one head is 64 rows of 256 contiguous bytes; 16 threads cover a row with 16-byte loads, 16 row
// groups cover the block, so every warp load instruction reads two full 256-byte rows.
// Outputs per (b, h, j): Qbar, Kbar (FP32 means over the valid tokens), BF16 copies of Kbar and
// of the value mean Vbar (surrogate MMA operands), and optionally the two 32-token anchor means of Q.
// -------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) summary_kernel(const __nv_bfloat16* __restrict__ q,
                                                      const __nv_bfloat16* __restrict__ k,
                                                      const __nv_bfloat16* __restrict__ v, Shape s, Work w,
                                                      int anchors) {
  __shared__ float red[8][4][kHeadDim];
  const int j = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c16 = tid & 15, rg = tid >> 4;
  const int t0 = j * kBlock;
  const int n = min(kBlock, s.N - t0);
  const int nlo = min(n, kAnchor), nhi = n - nlo;

  for (int h = 0; h < s.H; ++h) {
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
      w.qbar[o] = (sqlo + sqhi) / fn;
      w.kbar[o] = kb;
      w.kbar_h[o] = __float2bfloat16_rn(kb);
      w.vbar_h[o] = __float2bfloat16_rn(sv / fn);
      if (anchors) {
        const size_t a0 = (bh * s.Na + 2 * (size_t)j) * kHeadDim + c;
        w.qanchor[a0] = sqlo / (float)nlo;
        if (nhi > 0) w.qanchor[a0 + kHeadDim] = sqhi / (float)nhi;
      }
    }
    __syncthreads();
  }
}

// -------------------------------------------------------------------------------------------------
// Threshold statistics (Eq. (5)), FP64 accumulation.  kmean = mean_j Kbar_j and the centred
// covariance C = mean_j (Kbar_j - kmean)(Kbar_j - kmean)^T, so that
// sigma_i^2 = s^2 Qbar_i C Qbar_i^T equals Eq. (5)'s second moment minus mu_i^2 without cancellation.
// Grid (8, BH): each CTA produces 16 rows of C (and all CTAs recompute kmean, which is cheap).
// -------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) kstats_kernel(Shape s, Work w) {
  __shared__ double mk[kHeadDim];
  __shared__ double xs[32][kHeadDim];
  const int bh = blockIdx.y, tid = threadIdx.x;
  const float* kb = w.kbar + (size_t)bh * s.Nb * kHeadDim;
  if (tid < kHeadDim) {
    double acc = 0.0;
    for (int j = 0; j < s.Nb; ++j) acc += (double)kb[(size_t)j * kHeadDim + tid];
    mk[tid] = acc / s.Nb;
    if (blockIdx.x == 0) w.kmean[(size_t)bh * kHeadDim + tid] = acc / s.Nb;
  }
  __syncthreads();
  const int r = 16 * blockIdx.x + (tid >> 4);
  const int c0 = (tid & 15) * 8;
  double acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0;
  for (int j0 = 0; j0 < s.Nb; j0 += 32) {
    const int nj = min(32, s.Nb - j0);
    for (int idx = tid; idx < nj * kHeadDim; idx += 256) {
      const int jj = idx / kHeadDim, c = idx % kHeadDim;
      xs[jj][c] = (double)kb[(size_t)(j0 + jj) * kHeadDim + c] - mk[c];
    }
    __syncthreads();
    for (int jj = 0; jj < nj; ++jj) {
      const double xr = xs[jj][r];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += xr * xs[jj][c0 + e];
    }
    __syncthreads();
  }
  float* cov = w.kcov + (size_t)bh * kHeadDim * kHeadDim;
#pragma unroll
  for (int e = 0; e < 8; ++e) cov[r * kHeadDim + c0 + e] = (float)(acc[e] / s.Nb);
}

// -------------------------------------------------------------------------------------------------
// tau_i = mu_i + tau * sigma_i with mu_i = s Qbar_i . kmean, sigma_i^2 = s^2 Qbar_i C Qbar_i^T (FP64),
// stored rounded to FP32, the precision the routing comparison is made in.
// Grid (ceil(Nb / 64), BH), 8 warps x 8 rows.
// -------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) thresh_kernel(Shape s, Work w, float tau) {
  extern __shared__ float cov_s[];  // [128][128]
  __shared__ double qrow[8][kHeadDim];
  const int bh = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* cov = w.kcov + (size_t)bh * kHeadDim * kHeadDim;
  for (int idx = tid; idx < kHeadDim * kHeadDim / 4; idx += 256)
    reinterpret_cast<float4*>(cov_s)[idx] = reinterpret_cast<const float4*>(cov)[idx];
  __syncthreads();
  const double* mk = w.kmean + (size_t)bh * kHeadDim;
  for (int rr = 0; rr < 8; ++rr) {
    const int i = blockIdx.x * 64 + warp * 8 + rr;
    if (i >= s.Nb) break;
    const float* qb = w.qbar + ((size_t)bh * s.Nb + i) * kHeadDim;
    double mu = 0.0;
    for (int c = lane; c < kHeadDim; c += 32) {
      const double x = (double)qb[c];
      qrow[warp][c] = x;
      mu += x * mk[c];
    }
    __syncwarp();
    double quad = 0.0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = lane + 32 * e;
      double y = 0.0;
      for (int d = 0; d < kHeadDim; ++d) y += (double)cov_s[d * kHeadDim + c] * qrow[warp][d];
      quad += y * qrow[warp][c];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mu += __shfl_xor_sync(0xffffffffu, mu, o);
      quad += __shfl_xor_sync(0xffffffffu, quad, o);
    }
    if (lane == 0) {
      const double sd = (double)kScale;
      const double m = sd * mu;
      const double var = fmax(sd * sd * quad, 0.0);
      w.thresh[(size_t)bh * s.Nb + i] = (float)(m + (double)tau * sqrt(var));
    }
    __syncwarp();
  }
}

// -------------------------------------------------------------------------------------------------
// Routing: bit j of row i is set iff s_ij = s * Qbar_i . Kbar_j > tau_i (FP32), |i - j| <= 1, or
// block j overlaps the sink.  The proxies are consumed as they are produced (only the bitmask and
// per-row counts reach memory).  Grid (ceil(Nb / 64), BH); a 64 x 64 tile of proxies per step,
// 4 x 4 per thread from transposed shared-memory tiles.
// -------------------------------------------------------------------------------------------------
constexpr int kRoutePad = 68;

__global__ void __launch_bounds__(256) route_kernel(Shape s, Work w, int sink_b0, int sink_b1) {
  extern __shared__ float rsm[];
  float* Qt = rsm;                      // [128][68]
  float* Kt = rsm + kHeadDim * kRoutePad;  // [128][68]
  __shared__ float th[64];
  __shared__ int cnt[64];
  const int bh = blockIdx.y, i0 = blockIdx.x * 64, tid = threadIdx.x, lane = tid & 31;
  const int ti = tid >> 4, tj = tid & 15;
  const float* qb = w.qbar + (size_t)bh * s.Nb * kHeadDim;
  const float* kb = w.kbar + (size_t)bh * s.Nb * kHeadDim;
  for (int idx = tid; idx < 64 * kHeadDim; idx += 256) {
    const int r = idx / kHeadDim, c = idx % kHeadDim;
    Qt[c * kRoutePad + r] = (i0 + r < s.Nb) ? qb[(size_t)(i0 + r) * kHeadDim + c] : 0.f;
  }
  if (tid < 64) {
    th[tid] = (i0 + tid < s.Nb) ? w.thresh[(size_t)bh * s.Nb + i0 + tid] : 0.f;
    cnt[tid] = 0;
  }
  for (int j0 = 0; j0 < s.Nb; j0 += 64) {
    __syncthreads();
    for (int idx = tid; idx < 64 * kHeadDim; idx += 256) {
      const int r = idx / kHeadDim, c = idx % kHeadDim;
      Kt[c * kRoutePad + r] = (j0 + r < s.Nb) ? kb[(size_t)(j0 + r) * kHeadDim + c] : 0.f;
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
#pragma unroll 4
    for (int d = 0; d < kHeadDim; ++d) {
      const float4 qa = *reinterpret_cast<const float4*>(&Qt[d * kRoutePad + 4 * ti]);
      const float4 kk = *reinterpret_cast<const float4*>(&Kt[d * kRoutePad + 4 * tj]);
      const float av[4] = {qa.x, qa.y, qa.z, qa.w};
      const float bv[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(av[a], bv[c], acc[a][c]);
    }
    // 4 rows x 4 columns of decisions -> one nibble per row, OR-combined across the 8 lanes that
    // share a 32-column word.
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int il = 4 * ti + a;
      const int i = i0 + il;
      uint32_t bits = 0;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int jj = j0 + 4 * tj + c;
        const float shat = acc[a][c] * kScale;
        if (jj < s.Nb && shat > th[il]) bits |= 1u << (4 * (tj & 7) + c);
      }
      bits |= __shfl_xor_sync(0xffffffffu, bits, 1);
      bits |= __shfl_xor_sync(0xffffffffu, bits, 2);
      bits |= __shfl_xor_sync(0xffffffffu, bits, 4);
      if ((lane & 7) == 0 && i < s.Nb) {
        const int wd = (j0 >> 5) + (tj >> 3);
        if (wd < s.Nw) {
          const int jb = 32 * wd;
          for (int jj = max(i - 1, jb); jj <= min(i + 1, jb + 31); ++jj)
            if (jj >= 0 && jj < s.Nb) bits |= 1u << (jj - jb);
          if (sink_b0 <= sink_b1) {
            const int lo = max(sink_b0, jb), hi = min(sink_b1, jb + 31);
            for (int jj = lo; jj <= hi; ++jj) bits |= 1u << (jj - jb);
          }
          w.mask[((size_t)bh * s.Nb + i) * s.Nw + wd] = bits;
          atomicAdd(&cnt[il], __popc(bits));
        }
      }
    }
  }
  __syncthreads();
  if (tid < 64 && i0 + tid < s.Nb) {
    const int c = cnt[tid];
    w.rowcount[(size_t)bh * s.Nb + i0 + tid] = c;
    atomicAdd(&w.stats[0], (unsigned long long)c);
    atomicMin(&w.stats[1], (unsigned long long)c);
    atomicMax(&w.stats[2], (unsigned long long)c);
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

void launch_summary(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, const Shape& s,
                    const Work& w, bool anchors, cudaStream_t st) {
  summary_kernel<<<dim3(s.Nb, s.B), 256, 0, st>>>(q, k, v, s, w, anchors ? 1 : 0);
}

void launch_kstats(const Shape& s, const Work& w, cudaStream_t st) {
  kstats_kernel<<<dim3(kHeadDim / 16, s.BH), 256, 0, st>>>(s, w);
}

void launch_thresh(const Shape& s, const Work& w, float tau, cudaStream_t st) {
  const int smem = kHeadDim * kHeadDim * sizeof(float);
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(thresh_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    configured = true;
  }
  thresh_kernel<<<dim3((s.Nb + 63) / 64, s.BH), 256, smem, st>>>(s, w, tau);
}

void launch_route(const Shape& s, const Work& w, int sink_b0, int sink_b1, cudaStream_t st) {
  const int smem = 2 * kHeadDim * kRoutePad * sizeof(float);
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    configured = true;
  }
  route_kernel<<<dim3((s.Nb + 63) / 64, s.BH), 256, smem, st>>>(s, w, sink_b0, sink_b1);
}

void launch_expand_mask(const Shape& s, const Work& w, unsigned char* mask_out, cudaStream_t st) {
  expand_mask_kernel<<<1184, 256, 0, st>>>(s, w, mask_out);
}

}  // namespace sol
