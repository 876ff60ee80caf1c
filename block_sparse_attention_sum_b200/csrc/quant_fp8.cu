// E4M3 operands of the FP8 forward: V and the compressed keys / values here; Q and K are quantised
// by the block-summary kernels in their pass over Q and K (quant_block_rows in fp8.cuh).
//
// Sol-Attn2 draft, section "FP8 quantization and ExpCast": one scale per 64-token block for Q and K,
// one per head for V, s = max |X| / 448 (an all-zero block keeps s = 1), codes E4M3(X / s) rounded to
// nearest even with saturation.  The compressed keys and values of the surrogate take the same
// rules: the block means Kbar_j as a key array (one scale per 64 consecutive means of a head) and
// the value means Vbar_j = Vhat_j / n_j with the head's V scale.
//
// Layouts (all E4M3 bytes): Q8, K8, V8 in BTHD order like the inputs; Kbar8 and Vbar8 as
// [BH][Nbp][128] with Nbp = Nb rounded up to 128 (zero rows past Nb), so that one 128-row box covers
// any surrogate chunk.  Scales: sq, sk [BH][Nb]; skbar [BH][Nbp / 64]; sv [BH].
#include <cuda_bf16.h>
#include <cfloat>

#include "common.cuh"
#include "fp8.cuh"

namespace sol {

namespace {

__device__ __forceinline__ float block_max_256(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) m = fmaxf(m, red[i]);
  __syncthreads();
  return m;
}

// Thread layout of a 64 x 128 tile over 256 threads: 8 channels 8 (tid % 16) .. per thread, rows
// tid / 16 + 16 r for r = 0..3.
__device__ __forceinline__ void load_rows_bf16(const __nv_bfloat16* x, const Shape& s, int b, int h, int t0, int n,
                                               int tid, float (&v)[4][8], float* amax) {
  const int c16 = tid & 15, rg = tid >> 4;
  float m = 0.f;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int row = rg + 16 * r;
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (row < n)
      raw = *reinterpret_cast<const uint4*>(x + (((size_t)b * s.N + t0 + row) * s.H + h) * kHeadDim + 8 * c16);
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(p[e]);
      v[r][2 * e] = f.x;
      v[r][2 * e + 1] = f.y;
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
  *amax = m;
}

// grid (Nb, BH): V with the head's scale, and the block's value mean Vbar_j (FP32 column sums over
// its n_j tokens, divided by n_j) with the same scale into row j of Vbar8.
__global__ void __launch_bounds__(256) quant_v_kernel(const __nv_bfloat16* __restrict__ v, uint8_t* __restrict__ v8,
                                                      uint8_t* __restrict__ vbar8, float* __restrict__ sv,
                                                      const unsigned int* __restrict__ vmax, const Shape s, int Nbp) {
  __shared__ float colsum[16][kHeadDim];
  const int j = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int b = bh / s.H, h = bh % s.H, t0 = j * kBlock, n = min(kBlock, s.N - t0);
  const float m = __uint_as_float(vmax[bh]);
  const float sc = m > 0.f ? m / 448.0f : 1.0f;
  if (j == 0 && tid == 0) sv[bh] = sc;
  const Quot448 qc = quot448_setup(m > 0.f ? m : 1.0f);
  float vals[4][8], amax;
  load_rows_bf16(v, s, b, h, t0, n, tid, vals, &amax);
  const int c16 = tid & 15, rg = tid >> 4;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int row = rg + 16 * r;
    if (row < n)
      *reinterpret_cast<uint2*>(v8 + (((size_t)b * s.N + t0 + row) * s.H + h) * kHeadDim + 8 * c16) =
          m > 0.f ? codes8(vals[r], qc) : make_uint2(0u, 0u);
  }
  // column sums: rows beyond n were loaded as zeros
#pragma unroll
  for (int e = 0; e < 8; ++e) colsum[rg][8 * c16 + e] = (vals[0][e] + vals[1][e]) + (vals[2][e] + vals[3][e]);
  __syncthreads();
  if (tid < kHeadDim / 2) {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int g = 0; g < 16; ++g) {
      a0 += colsum[g][2 * tid];
      a1 += colsum[g][2 * tid + 1];
    }
    const float inv_n = 1.0f / (float)n;
    const uint32_t w = m > 0.f ? to_e4m3x2(quot448(a0 * inv_n, qc), quot448(a1 * inv_n, qc)) : 0u;
    *reinterpret_cast<uint16_t*>(vbar8 + ((size_t)bh * Nbp + j) * kHeadDim + 2 * tid) = (uint16_t)w;
  }
}

// grid (Nbp / 64, BH): the block means Kbar (FP32) of 64 consecutive key blocks share one scale;
// rows past Nb are written as zeros in Kbar8 and Vbar8.
__global__ void __launch_bounds__(256) quant_kbar_kernel(const float* __restrict__ kbar, uint8_t* __restrict__ kbar8,
                                                         uint8_t* __restrict__ vbar8, float* __restrict__ skbar,
                                                         const Shape s, int Nbp) {
  __shared__ float red[8];
  const int g = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int c16 = tid & 15, rg = tid >> 4;
  float vals[4][8];
  float amax = 0.f;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int j = 64 * g + rg + 16 * r;
#pragma unroll
    for (int e = 0; e < 8; ++e) vals[r][e] = 0.f;
    if (j < s.Nb) {
      const float4* src = reinterpret_cast<const float4*>(kbar + ((size_t)bh * s.Nb + j) * kHeadDim + 8 * c16);
      const float4 a = src[0], c = src[1];
      vals[r][0] = a.x; vals[r][1] = a.y; vals[r][2] = a.z; vals[r][3] = a.w;
      vals[r][4] = c.x; vals[r][5] = c.y; vals[r][6] = c.z; vals[r][7] = c.w;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(vals[r][e]));
  }
  const float m = block_max_256(amax, red);
  const float sc = m > 0.f ? m / 448.0f : 1.0f;
  if (tid == 0) skbar[(size_t)bh * (Nbp / 64) + g] = sc;
  const Quot448 qc = quot448_setup(m > 0.f ? m : 1.0f);
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int j = 64 * g + rg + 16 * r;
    const size_t off = ((size_t)bh * Nbp + j) * kHeadDim + 8 * c16;
    *reinterpret_cast<uint2*>(kbar8 + off) = (j < s.Nb && m > 0.f) ? codes8(vals[r], qc) : make_uint2(0u, 0u);
    if (j >= s.Nb) *reinterpret_cast<uint2*>(vbar8 + off) = make_uint2(0u, 0u);
  }
}

}  // namespace

void launch_quant_fp8(const __nv_bfloat16* v, const Shape& s, const Work& w, const Fp8Work& f, cudaStream_t st) {
  const int nbp = fp8_rows_padded(s);
  quant_v_kernel<<<dim3(s.Nb, s.BH), 256, 0, st>>>(v, f.v8, f.vbar8, f.sv, f.vmax, s, nbp);
  quant_kbar_kernel<<<dim3(nbp / 64, s.BH), 256, 0, st>>>(w.kbar, f.kbar8, f.vbar8, f.skbar, s, nbp);
}

}  // namespace sol
