// E4M3 tensor-core products and the ExpCast encoder of the FP8 forward.
//
// Sol-Attn2 draft, section "FP8 quantization and ExpCast": Q and K carry one E4M3 scale per 64-token
// block, V one per head (s = max |X| / 448); QK and PV run on FP8 operands with FP32 accumulation;
// ExpCast turns a base-2 score u relative to the shared pivot into the E4M3 probability byte
// c(u) = clip_[0,120](RNE(8u + 55.65)), whose decoded value is about 2^u.
#pragma once
#include <cstdint>
#include <cmath>
#ifdef __CUDACC__
#include <cuda_bf16.h>
#endif

namespace sol {

// ExpCast constants: offset of the code line and the largest code (E4M3 0x78 = 2^8).
constexpr float kExpCastOffset = 55.65f;
constexpr int kExpCastMaxCode = 120;

// The code of base-2 score x * fs against the integer pivot `pivot`, as the kernel computes it:
// v = fma(x, 8 fs, 55.65 - 8 pivot) (one rounding), clamped below at 0, rounded to the nearest
// integer (ties to even) by adding 1.5 * 2^23, whose unit in the last place is 1: the rounded value
// is then the low byte of the sum's bit pattern.  The clip at 120 is not applied: the pivot rule
// keeps x * fs <= pivot + 8, so v <= 119.65 up to the FP32 rounding of the products.  A masked
// score (x = -inf) gives code 0, the E4M3 encoding of +0.
__host__ __device__ __forceinline__ uint32_t expcast_code_f32(float x, float f8, float c) {
  float v = fmaf(x, f8, c);
  v = fmaxf(v, 0.0f);
  const float r = v + 12582912.0f;
  uint32_t bits;
#ifdef __CUDA_ARCH__
  bits = __float_as_uint(r);
#else
  __builtin_memcpy(&bits, &r, 4);
#endif
  return bits & 0xffu;
}

// Four codes in one 32-bit word, the first key in the low byte: the layout of an E4M3 A operand in
// tensor memory (one row per lane, four consecutive K elements per 32-bit column).
__host__ __device__ __forceinline__ uint32_t pack_codes4(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3) {
  return c0 | (c1 << 8) | (c2 << 16) | (c3 << 24);
}

// 2^k for an integer-valued float k (exact; 0 below the normal range, k = -inf included).
__host__ __device__ __forceinline__ float pow2i(float k) {
  if (!(k >= -126.0f)) return 0.0f;
  const int e = (int)k + 127;
  const uint32_t bits = (uint32_t)(e > 254 ? 254 : e) << 23;
  float r;
#ifdef __CUDA_ARCH__
  r = __uint_as_float(bits);
#else
  __builtin_memcpy(&r, &bits, 4);
#endif
  return r;
}

// X / s for s = m / 448 (m = max |X| > 0 of the scale's group), as the quantisers evaluate it:
// RN(RN(x * 448) / m) without a division per element.  With s2 = 2^(127 - E) (E the biased
// exponent of m) scaling changes no rounding, so the value is RN(a / m2) for a = RN(x * 448 s2)
// and m2 = m s2 in [1, 2).  With y = RN(1 / m2), q = RN(a y) lies within one unit in the last place
// of a / m2, the remainder a - q m2 is exact in one FMA, and RN(q + (a - q m2) y) is the correctly
// rounded quotient (Markstein's theorem, the correction step of the IA-64 division sequences).
// Outside 2^-100 <= m < 2^101 the division is taken as written.  The sign is copied from x, so
// -0 stays -0 as in the division.
struct Quot448 {
  float k448;   // 448 s2
  float m2;     // m s2
  float y;      // RN(1 / m2)
  float m;      // m itself, for the division outside the range
  bool fast;
};

__host__ __device__ __forceinline__ Quot448 quot448_setup(float m) {
  uint32_t bits;
#ifdef __CUDA_ARCH__
  bits = __float_as_uint(m);
#else
  __builtin_memcpy(&bits, &m, 4);
#endif
  const uint32_t eb = (bits >> 23) & 0xffu;
  Quot448 c;
  c.m = m;
  c.fast = eb >= 27u && eb <= 227u;
  const uint32_t sbits = (254u - (c.fast ? eb : 127u)) << 23;   // 2^(127 - E)
  float s2;
#ifdef __CUDA_ARCH__
  s2 = __uint_as_float(sbits);
#else
  __builtin_memcpy(&s2, &sbits, 4);
#endif
  c.k448 = 448.0f * s2;
  c.m2 = m * s2;
  c.y = 1.0f / c.m2;
  return c;
}

__host__ __device__ __forceinline__ float quot448(float x, const Quot448& c) {
  if (!c.fast) return (x * 448.0f) / c.m;
  const float a = x * c.k448;
  const float q = a * c.y;
  const float r = fmaf(-q, c.m2, a);
  return copysignf(fmaf(r, c.y, q), x);
}

// Pivot rule of the online softmax: the pivot is an integer (base 2) and moves only when the running
// maximum exceeds it by more than 8, to ceil(max) - 8, so that every coded score satisfies u <= 8.
// Returns the new pivot; *alpha = 2^(old - new) rescales what was accumulated against the old one
// (0 when there was none).
__host__ __device__ __forceinline__ float pivot_update(float pivot, float mx, float* alpha, bool* moved) {
  if (mx > pivot + 8.0f) {
    const float np = ceilf(mx) - 8.0f;
    *alpha = pow2i(pivot - np);
    *moved = true;
    return np;
  }
  *alpha = 1.0f;
  *moved = false;
  return pivot;
}

#ifdef __CUDACC__
// Instruction descriptor, kind::f8f6f4: E4M3 A and B (format 0), FP32 accumulator, M x N tile.
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (0u << 7) | (0u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem], E4M3 operands, K = 32 per instruction; one thread issues.
__device__ __forceinline__ void umma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]: A (M x K, E4M3) from tensor memory, one row per lane, four K
// elements per 32-bit column (lowest K index in the low byte).
__device__ __forceinline__ void umma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// One column per thread (32 lanes x 32 bit).
__device__ __forceinline__ uint32_t tmem_ld1(uint32_t taddr) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
  return r;
}
__device__ __forceinline__ void tmem_st1(uint32_t taddr, uint32_t r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(r) : "memory");
}

// Two FP32 values to two E4M3 bytes (round to nearest even, saturating at +-448), lo in the low byte.
__device__ __forceinline__ uint32_t to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// X / s is evaluated as (x * 448) / m (quot448): for a BF16 x the product is exact and the
// quotient correctly rounded, so a value that lies exactly halfway between two E4M3 numbers
// (frequent: x and m share most of their few mantissa bits) stays exactly halfway and rounds to
// even, as the definition asks; x / fl(m / 448) can land just off the midpoint and round the
// other way.

// quot448 of two values on f32x2 lanes (each lane rounds as the scalar instruction does, so the
// pair equals two quot448 calls bit for bit); c.fast must hold.
__device__ __forceinline__ float2 quot448x2(float x0, float x1, const Quot448& c) {
  uint64_t x, k, y, m2, a, q, r, o;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(x0), "f"(x1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(k) : "f"(c.k448));
  asm("mov.b64 %0, {%1, %1};" : "=l"(y) : "f"(c.y));
  asm("mov.b64 %0, {%1, %1};" : "=l"(m2) : "f"(-c.m2));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(a) : "l"(x), "l"(k));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(q) : "l"(a), "l"(y));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(q), "l"(m2), "l"(a));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(o) : "l"(r), "l"(y), "l"(q));
  float2 res;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(res.x), "=f"(res.y) : "l"(o));
  return make_float2(copysignf(res.x, x0), copysignf(res.y, x1));
}

// Eight values of a block with maximum |X| = m > 0 (c = quot448_setup(m)), as four E4M3 pairs in
// one 8-byte word.
__device__ __forceinline__ uint2 codes8(const float (&v)[8], const Quot448& c) {
  uint32_t w[4];
  if (c.fast) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 q = quot448x2(v[2 * e], v[2 * e + 1], c);
      w[e] = to_e4m3x2(q.x, q.y);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) w[e] = to_e4m3x2(quot448(v[2 * e], c), quot448(v[2 * e + 1], c));
  }
  return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// This thread's largest |x| over its four rows of 8 BF16 channels (`rows`, as the block-summary
// kernels load them).
__device__ __forceinline__ float thread_absmax(const uint4 (&rows)[4]) {
  float m = 0.f;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&rows[r]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(p[e]);
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
  return m;
}

// Block-wide maxima (256 threads) of kT per-thread values, all in one pass: warp shuffles, then the
// eight warp maxima of each value through `red` (8 kT floats of shared memory).  The caller puts a
// block synchronisation between the two halves, shared with its other reductions.
template <int kT>
__device__ __forceinline__ void block_max_post(float (&m)[kT], float* red) {
#pragma unroll
  for (int t = 0; t < kT; ++t) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m[t] = fmaxf(m[t], __shfl_xor_sync(0xffffffffu, m[t], o));
  }
  if ((threadIdx.x & 31) == 0) {
#pragma unroll
    for (int t = 0; t < kT; ++t) red[8 * t + (threadIdx.x >> 5)] = m[t];
  }
}
template <int kT>
__device__ __forceinline__ void block_max_collect(float (&m)[kT], const float* red) {
#pragma unroll
  for (int t = 0; t < kT; ++t) {
    float b = red[8 * t];
#pragma unroll
    for (int i = 1; i < 8; ++i) b = fmaxf(b, red[8 * t + i]);
    m[t] = b;
  }
}

// E4M3 codes of one 64-token block (one scale, s = max |X| / 448; an all-zero block keeps s = 1 and
// zero codes) from the rows the block-summary kernels hold: this thread's rows rg + 16 r (r < 4) of
// channels 8 c16 .. 8 c16 + 7, written to x8 ([B][N][H][128] bytes) and the scale to *scale (by
// thread 0).  Rows past the sequence (row >= n) are not written.
__device__ __forceinline__ void quant_block_rows(const uint4 (&rows)[4], float m, uint8_t* x8, float* scale, int N,
                                                 int H, int b, int h, int t0, int n, int tid) {
  const int c16 = tid & 15, rg = tid >> 4;
  if (tid == 0) *scale = m > 0.f ? m / 448.0f : 1.0f;
  const Quot448 qc = quot448_setup(m > 0.f ? m : 1.0f);
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int row = rg + 16 * r;
    if (row >= n) continue;
    float v[8];
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&rows[r]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(p[e]);
      v[2 * e] = f.x;
      v[2 * e + 1] = f.y;
    }
    *reinterpret_cast<uint2*>(x8 + (((size_t)b * N + t0 + row) * H + h) * 128 + 8 * c16) =
        m > 0.f ? codes8(v, qc) : make_uint2(0u, 0u);
  }
}
#endif  // __CUDACC__

}  // namespace sol
