// Split-KV combine.  With kv_splits = S > 1 the fused kernel runs S CTAs per 128-row query tile,
// each over a contiguous share of the tile's key tiles (exact tiles first, then the surrogate
// tiles), and writes its partial online-softmax state per query row: the base-2 reference m_s, the
// row sum l_s and the unnormalised accumulator O_s.  The parts of a row merge exactly as two halves
// of one softmax do:
//   o = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s,   M = max_s m_s,
// a split that saw no key (m_s = -inf) contributing nothing.  The pages' kernels expose this as a
// kv_splits tuning knob (Sol-Attn README, "Long-sequence tuning on H100").
#include <cfloat>

#include "common.cuh"

namespace sol {

// One warp per query row: lane l owns channels 4l .. 4l + 3.
__global__ void __launch_bounds__(256) splitkv_combine_kernel(Shape s, int splits, int rows_pad,
                                                              const float* __restrict__ part_o,
                                                              const float* __restrict__ part_ml,
                                                              __nv_bfloat16* __restrict__ out, int row_lo,
                                                              int row_hi) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp, bh = blockIdx.y;
  if (row >= rows_pad || row < row_lo || row >= row_hi) return;
  const size_t per_split = (size_t)s.BH * rows_pad;
  const size_t r = (size_t)bh * rows_pad + row;
  float M = -INFINITY;
  for (int sp = 0; sp < splits; ++sp) M = fmaxf(M, part_ml[2 * (sp * per_split + r)]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float den = 0.f;
  for (int sp = 0; sp < splits; ++sp) {
    const size_t idx = sp * per_split + r;
    const float m = part_ml[2 * idx];
    if (m == -INFINITY) continue;   // no key in this split: weight 0 (its O is not read)
    float wgt;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(wgt) : "f"(m - M));
    den = fmaf(wgt, part_ml[2 * idx + 1], den);
    const float4 o = *reinterpret_cast<const float4*>(part_o + idx * kHeadDim + 4 * lane);
    acc.x = fmaf(wgt, o.x, acc.x);
    acc.y = fmaf(wgt, o.y, acc.y);
    acc.z = fmaf(wgt, o.z, acc.z);
    acc.w = fmaf(wgt, o.w, acc.w);
  }
  const float inv = 1.f / den;
  const int b = bh / s.H, h = bh % s.H;
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  uint2 packed;
  packed.x = *reinterpret_cast<uint32_t*>(&lo);
  packed.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(out + (((size_t)b * s.N + row) * s.H + h) * kHeadDim + 4 * lane) = packed;
}

void launch_splitkv_combine(const Shape& s, int splits, const float* part_o, const float* part_ml,
                            __nv_bfloat16* out, int row_lo, int row_hi, cudaStream_t st) {
  const int rows_pad = s.QT * 128;
  splitkv_combine_kernel<<<dim3((rows_pad + 7) / 8, s.BH), 256, 0, st>>>(s, splits, rows_pad, part_o, part_ml, out,
                                                                         row_lo, row_hi);
}

}  // namespace sol
