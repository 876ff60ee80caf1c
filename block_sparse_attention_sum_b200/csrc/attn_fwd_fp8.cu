// Fused FP8 (E4M3) + ExpCast forward for sm_100a: the pipeline of the BF16 kernel with E4M3
// operands, ExpCast probability bytes and the row sums taken by the tensor cores.
//
// Sol-Attn2 draft, section "FP8 quantization and ExpCast": Q and K carry one E4M3 scale per 64-token
// block and V one per head; QK and PV use FP8 operands with FP32 accumulation and the scales restore
// the magnitudes; the compressed keys keep their mass through an additive bias; ExpCast gives the
// probability byte c(u) = clip_[0,120](RNE(8u + 55.65)) of a base-2 score u relative to a shared
// online pivot, and the same decoded weights enter the PV product and the denominator.
// Sol-Attn paper (arXiv 2607.24027), section 3.2, for the exact / surrogate split; Sol-Attn2 draft,
// "Routing and complementary approximation", for the tail merged in the epilogue.
//
// Differences from the BF16 kernel:
//  * Operands: Q8 and K8 tiles are 128 rows x 128 bytes (one 128-byte swizzle row per token), so
//    S = Q K^T is four K = 32 kind::f8f6f4 products.  V8 stays in BTHD order and is the MN-major B
//    operand of O += P V (keys in 8-row groups, 128 channels per row).  Surrogate tiles read the
//    E4M3 compressed keys / values (Kbar8, Vbar8) in the same formats.
//  * Scales: the producer writes the key operand's two 64-row scales into the tile descriptor;
//    the softmax folds s_Q s_K / sqrt(128) log2 e into one multiplier per row and half-tile.
//  * Softmax: a score's code is one saturating FMA (on the score scaled by 2^-7, so the
//    saturation is the clamp at 0) and an add of 1.5 * 2^16 on paired f32x2 lanes, whose low byte
//    is the rounded code; four codes per 32-bit TMEM column (P of a warpgroup: 64 keys in 16
//    columns), gathered by byte permutes.  No exponential, no row sum on the CUDA cores.  The
//    kernel is bound by this instruction stream, not by the tensor cores.
//  * Row sums: the P V product runs with N = 144, its B operand's channels 128..143 being E4M3 ones,
//    so the same instruction accumulates the sum of the decoded weights in TMEM (L_w) beside O_w:
//    the denominator is exactly the FP32 sum of the weights the P V product used (sums of E4M3
//    weights are exact in FP32 at these sizes); it is rescaled with O when the pivot moves.
//  * Pivot: an integer in base 2, moved only when the running maximum exceeds it by more than 8, to
//    ceil(max) - 8 (every coded score then has u <= 8, so the clip at 120 never acts); rescale
//    factors are exact powers of two.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cfloat>

#include "attn_fwd_fp8.cuh"
#include "fp8.cuh"
#include "ptx.cuh"

namespace sol {

namespace {

constexpr int kStages = 4;                  // K / V ring depth
constexpr int kDescRing = 8;                // tile descriptors in flight
constexpr uint32_t kTile8 = 128 * 128;      // 128 rows x 128 E4M3 channels (16 KB), one swizzled tile
constexpr uint32_t kBox8 = 64 * 128;        // one 64-row box (8 KB)
// TMEM columns: S (128 x 128 FP32); P double buffer (per buffer 32 columns: warpgroup w's 64 keys
// as E4M3 codes in columns 16 w .. 16 w + 15); per warpgroup one N = 144 accumulator at
// kColO + kOStride w: O_w in its first 128 columns and the row sum L_w in the next 16 (all equal).
constexpr uint32_t kColS = 0, kColP = 128, kColO = 192, kOStride = 160;

enum : uint32_t { kTilePair = 0, kTileSingle = 1, kTilePooled = 2 };

struct TileDesc8 {
  uint32_t kind;
  int j0, j1;       // key blocks (exact tiles) or the surrogate chunk index (j0)
  uint32_t flags;   // bit 0/1: j0 exact for half 0/1; bit 2/3: j1 exact for half 0/1; bit 8: last tile
  float s0, s1;     // E4M3 scales of the key operand's rows 0..63 and 64..127
};

struct __align__(1024) Fp8Smem {
  uint8_t q[kTile8];               // 128 query rows x 128 channels, K-major SW128
  uint8_t k[kStages][kTile8];      // 128 keys x 128 channels, K-major SW128
  uint8_t v[kStages][kTile8];      // 128 keys x 128 channels: MN-major SW128 B operand of P V
  uint8_t ones[32 * 128];          // E4M3 1.0 (0x38): channels 128..143 of the P V product's B operand
  TileDesc8 desc[kDescRing];
  uint64_t kfull[kStages], kempty[kStages], vfull[kStages], vempty[kStages];
  uint64_t dfull[kDescRing];
  uint64_t qfull, sfull, sread, pready[2], pvdone[2], mmadone, mmadone2;
  uint64_t lbar;
  float xm[2][128], xl[2][128];    // [warpgroup][row] pivot and row sum, for the epilogue merge
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytes = sizeof(Fp8Smem);
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(offsetof(Fp8Smem, ones) % 1024 == 0, "swizzled operands must be 1024-byte aligned");

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Two E4M3 bytes (low byte first) to two floats (exact: E4M3 values are FP16 values).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t two) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(two));
  return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}

// Packed FP32 pairs (sm_100 f32x2 arithmetic: each lane rounds as the scalar instruction does).
__device__ __forceinline__ uint64_t f2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 unf2(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float r;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Four ExpCast codes packed first-key-lowest, bit for bit those of expcast_code_f32 / pack_codes4.
// The caller passes f8 / 128 and c0 / 128: scaling by a power of two commutes with rounding, so the
// saturating FMA yields max(RN(x f8 + c0), 0) / 128 and does the clamp at 0 in the same
// instruction (codes stay below 128: the pivot rule keeps u <= 8, so y <= 119.65).  Adding
// 1.5 * 2^16 (unit in the last place 2^-7) on f32x2 lanes rounds 128 y' to the nearest even
// integer in the low bits; three byte permutes gather the four low bytes.
__device__ __forceinline__ uint32_t expcast_pack4(float x0, float x1, float x2, float x3, float f8s, float c0s) {
  const uint64_t magic2 = f2(98304.0f, 98304.0f);
  const float2 ra = unf2(add2(f2(fma_sat(x0, f8s, c0s), fma_sat(x1, f8s, c0s)), magic2));
  const float2 rb = unf2(add2(f2(fma_sat(x2, f8s, c0s), fma_sat(x3, f8s, c0s)), magic2));
  const uint32_t lo = prmt(__float_as_uint(ra.x), __float_as_uint(ra.y), 0x0040u);
  const uint32_t hi = prmt(__float_as_uint(rb.x), __float_as_uint(rb.y), 0x0040u);
  return prmt(lo, hi, 0x5410u);
}

__device__ __forceinline__ void set_timeout(int* status) { atomicExch(status, kDevTimeout); }

// Debug builds (-DSOL_ATTN_DEBUG_BOUNDS) check every TMA tile coordinate against the tensor it
// reads; a failed check records kDevBounds and the copy is skipped (its consumer then runs out its
// bounded wait).  Release builds compile the checks away.
__device__ __forceinline__ bool tile_ok(uint32_t kind, int j0, int j1, int Nb, int* status) {
#ifdef SOL_ATTN_DEBUG_BOUNDS
  const bool ok = kind == 2u ? (j0 >= 0 && 128 * j0 < Nb)
                             : (j0 >= 0 && j0 < Nb && (kind != 0u || (j1 > j0 && j1 < Nb)));
  if (!ok) atomicExch(status, kDevBounds);
  return ok;
#else
  (void)kind; (void)j0; (void)j1; (void)Nb; (void)status;
  return true;
#endif
}

}  // namespace

template <bool kSol2>
__global__ void __launch_bounds__(384, 1)
    attn_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kp,
                        const __grid_constant__ CUtensorMap tm_vp, const FwdParams p, const Fp8Params f) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_u32(smem_raw) & 1023u) {   // uniform across the CTA
    if (tid == 0) atomicExch(p.status, kDevMisaligned);
    return;
  }
  Fp8Smem& sm = *reinterpret_cast<Fp8Smem*>(smem_raw);
  volatile int* abort = &sm.abort;

  const int unit = (int)blockIdx.x;
  const int bh = unit / p.qt_count, qt = p.qt_begin + unit % p.qt_count;
  const int b = bh / p.H, h = bh % p.H;
  const int qb0 = 2 * qt;
  const bool has_hi = qb0 + 1 < p.Nb;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kfull[s], 1);
      mbar_init(&sm.kempty[s], 1);
      mbar_init(&sm.vfull[s], 1);
      mbar_init(&sm.vempty[s], 1);
    }
    for (int s = 0; s < kDescRing; ++s) mbar_init(&sm.dfull[s], 1);
    mbar_init(&sm.qfull, 1);
    mbar_init(&sm.sfull, 1);
    mbar_init(&sm.sread, 256);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.pready[i], 128);
      mbar_init(&sm.pvdone[i], 1);
    }
    mbar_init(&sm.mmadone, 1);
    mbar_init(&sm.mmadone2, 1);
    mbar_init(&sm.lbar, 256);
    sm.abort = 0;
    fence_mbar_init();
  }
  {
    uint32_t* ones = reinterpret_cast<uint32_t*>(sm.ones);
    for (int i = tid; i < 32 * 128 / 4; i += 384) ones[i] = 0x38383838u;
    fence_async_smem();   // generic-proxy writes, read by the tensor cores
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
    // ----------------------------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      if (!kSol2) {
        tma_prefetch_desc(&tm_kp);
        tma_prefetch_desc(&tm_vp);
      }
      mbar_arrive_expect_tx(&sm.qfull, 2 * kBox8);
      if (tile_ok(1u, qb0, 0, p.Nb, p.status))
        for (int hf = 0; hf < 2; ++hf) tma_load_4d(&sm.q[hf * kBox8], &tm_q, &sm.qfull, 0, h, 64 * (qb0 + hf), b);

      const uint32_t* row0 = p.mask + ((size_t)bh * p.Nb + qb0) * p.Nw;
      const uint32_t* row1 = row0 + p.Nw;
      const float* sk = f.sk + (size_t)bh * p.Nb;
      const float* skbar = f.skbar + (size_t)bh * f.gk;
      int t = 0;
      bool ok = true;
      TileDesc8 prev;
      bool have_prev = false;
      auto issue = [&](TileDesc8 d) {
        const int s = t % kStages;
        const uint32_t ph = ((t / kStages) - 1) & 1;
        if (t >= kStages && !mbar_wait(&sm.kempty[s], ph, abort)) {
          ok = false;
          return;
        }
        sm.desc[t % kDescRing] = d;
        mbar_arrive(&sm.dfull[t % kDescRing]);
        const bool pooled = d.kind == kTilePooled;
        const int nblk = d.kind == kTilePair ? 2 : 1;
        mbar_arrive_expect_tx(&sm.kfull[s], pooled ? kTile8 : kBox8 * nblk);
        if (!tile_ok(d.kind, d.j0, d.j1, p.Nb, p.status)) {
        } else if (pooled) {
          tma_load_3d(&sm.k[s][0], &tm_kp, &sm.kfull[s], 0, 128 * d.j0, bh);
        } else {
          for (int slot = 0; slot < nblk; ++slot)
            tma_load_4d(&sm.k[s][slot * kBox8], &tm_k, &sm.kfull[s], 0, h, 64 * (slot ? d.j1 : d.j0), b);
        }
        ++t;
      };
      auto push = [&](TileDesc8 d) {
        if (have_prev && ok) issue(prev);
        prev = d;
        have_prev = true;
      };
      // exact tiles: the union of the two rows' exact blocks, in increasing order, two per tile
      int pend = -1;
      uint32_t pend_fl = 0;
      for (int wd = 0; wd < p.Nw && ok; ++wd) {
        const uint32_t a = row0[wd];
        const uint32_t c = has_hi ? row1[wd] : 0u;
        uint32_t u = a | c;
        while (u && ok) {
          const int bit = __ffs(u) - 1;
          u &= u - 1;
          const int j = 32 * wd + bit;
          const uint32_t fl = ((a >> bit) & 1u) | (((c >> bit) & 1u) << 1);
          if (pend < 0) {
            pend = j;
            pend_fl = fl;
          } else {
            push(TileDesc8{kTilePair, pend, j, pend_fl | (fl << 2), sk[pend], sk[j]});
            pend = -1;
          }
        }
      }
      if (pend >= 0 && ok) push(TileDesc8{kTileSingle, pend, pend, pend_fl, sk[pend], 1.0f});
      if (!kSol2) {
        // surrogate tiles: 128 compressed keys each; skip chunks that are exact for both rows
        const int nchunk = (p.Nb + 127) / 128;
        for (int ch = 0; ch < nchunk && ok; ++ch) {
          bool any = false;
          for (int e = 0; e < 4; ++e) {
            const int wd = 4 * ch + e;
            if (wd >= p.Nw) break;
            const int jb = 32 * wd;
            const int nvalid = min(32, p.Nb - jb);
            const uint32_t valid = nvalid >= 32 ? 0xffffffffu : ((1u << nvalid) - 1u);
            if ((~row0[wd] & valid) || (has_hi && (~row1[wd] & valid))) any = true;
          }
          if (any) push(TileDesc8{kTilePooled, ch, ch, 0u, skbar[2 * ch], skbar[2 * ch + 1]});
        }
      }
      if (have_prev && ok) {
        prev.flags |= 0x100u;
        issue(prev);
      }
      if (!ok) set_timeout(p.status);
      // never leave the CTA with bulk copies in flight
      for (int u = max(0, t - kStages); u < t; ++u) mbar_wait(&sm.kfull[u % kStages], (u / kStages) & 1, abort);
      mbar_wait(&sm.qfull, 0, abort);
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------------------------- S = Q K^T issuer
    if (lane == 0) {
      bool ok = mbar_wait(&sm.qfull, 0, abort);
      const uint32_t q_base = smem_u32(&sm.q[0]);
      for (int t = 0; ok; ++t) {
        const int s = t % kStages;
        if (!mbar_wait(&sm.kfull[s], (t / kStages) & 1, abort)) {
          ok = false;
          break;
        }
        const TileDesc8 d = sm.desc[t % kDescRing];
        // S still holds tile t - 1 until both softmax warpgroups have loaded it
        if (t >= 1 && !mbar_wait(&sm.sread, (t - 1) & 1, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int n = d.kind == kTileSingle ? 64 : 128;
        const uint32_t idesc = idesc_e4m3(128, n, false, false);
        const uint32_t k_base = smem_u32(&sm.k[s][0]);
        for (int kk = 0; kk < 4; ++kk)
          umma_ss_f8(tmem + kColS, sdesc_sw128(q_base + 32 * kk, 16, 1024), sdesc_sw128(k_base + 32 * kk, 16, 1024),
                     idesc, kk > 0 ? 1u : 0u);
        umma_commit(&sm.sfull);
        umma_commit(&sm.kempty[s]);
        if (d.flags & 0x100u) break;
      }
      if (!ok) set_timeout(p.status);
      umma_commit(&sm.mmadone);
      mbar_wait(&sm.mmadone, 0, abort);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------------- O += P V, L += P 1 issuer
    if (lane == 0) {
      bool ok = true;
      bool b_started = false;
      // N = 144: channels 0..127 are V, channels 128..143 a second 128-byte atom of the MN-major
      // operand, placed (by its leading byte offset) on a block of E4M3 ones, so the product's last 16
      // columns accumulate the row sums of the decoded weights in the same instruction
      const uint32_t idesc_pv = idesc_e4m3(128, 144, false, true);
      const uint32_t ones_base = smem_u32(&sm.ones[0]);
      for (int u = 0; ok; ++u) {
        const int s = u % kStages;
        const int bsel = u & 1;
        if (!mbar_wait(&sm.dfull[u % kDescRing], (u / kDescRing) & 1, abort) ||
            !mbar_wait(&sm.vfull[s], (u / kStages) & 1, abort)) {
          ok = false;
          break;
        }
        const TileDesc8 d = sm.desc[u % kDescRing];
        const uint32_t v_base = smem_u32(&sm.v[s][0]);
        for (int w = 0; w < 2 && ok; ++w) {
          if (!mbar_wait(&sm.pready[w], u & 1, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const bool skip = (w == 1 && d.kind == kTileSingle);   // no keys in the second half
          if (!skip) {
            const uint32_t p_col = tmem + kColP + 32 * bsel + 16 * w;   // P_w: 64 keys in 16 columns
            for (int kk = 0; kk < 2; ++kk) {
              // keys 64 w + 32 kk .. + 31: four 8-row groups of the MN-major V tile
              const uint32_t vs = v_base + w * kBox8 + kk * 4096;
              const uint64_t bd = sdesc_sw128(vs, ones_base - vs, 1024);
              const bool acc = w == 0 ? (u > 0 || kk > 0) : (b_started || kk > 0);
              umma_ts_f8(tmem + kColO + kOStride * w, p_col + 8 * kk, bd, idesc_pv, acc ? 1u : 0u);
            }
            if (w == 1) b_started = true;
          }
          umma_commit(&sm.pvdone[w]);
        }
        if (!ok) break;
        umma_commit(&sm.vempty[s]);
        if (d.flags & 0x100u) break;
      }
      if (!ok) set_timeout(p.status);
      umma_commit(&sm.mmadone2);
      mbar_wait(&sm.mmadone2, 0, abort);
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------------------------------------ V producer
    if (lane == 0) {
      bool ok = true;
      int u = 0;
      for (;; ++u) {
        const int s = u % kStages;
        if (!mbar_wait(&sm.dfull[u % kDescRing], (u / kDescRing) & 1, abort) ||
            (u >= kStages && !mbar_wait(&sm.vempty[s], ((u / kStages) - 1) & 1, abort))) {
          ok = false;
          break;
        }
        const TileDesc8 d = sm.desc[u % kDescRing];
        const bool pooled = d.kind == kTilePooled;
        const int nblk = d.kind == kTilePair ? 2 : 1;
        mbar_arrive_expect_tx(&sm.vfull[s], pooled ? kTile8 : kBox8 * nblk);
        if (!tile_ok(d.kind, d.j0, d.j1, p.Nb, p.status)) {
        } else if (pooled) {
          tma_load_3d(&sm.v[s][0], &tm_vp, &sm.vfull[s], 0, 128 * d.j0, bh);
        } else {
          for (int slot = 0; slot < nblk; ++slot)
            tma_load_4d(&sm.v[s][slot * kBox8], &tm_v, &sm.vfull[s], 0, h, 64 * (slot ? d.j1 : d.j0), b);
        }
        if (d.flags & 0x100u) {
          ++u;
          break;
        }
      }
      if (!ok) set_timeout(p.status);
      for (int w = max(0, u - kStages); w < u; ++w) mbar_wait(&sm.vfull[w % kStages], (w / kStages) & 1, abort);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // --------------------------------------------------------------- softmax / correction / epilogue
    // Warpgroup wg owns columns 64 wg .. 64 wg + 63 of every tile, with its own pivot, O_wg and L_wg;
    // the two halves of a row are merged exactly in the epilogue.
    const int wg = (warp - 4) >> 2;
    const int r = ((warp & 3) << 5) | lane;   // query row within the tile == TMEM lane
    const int hf = r >> 6;
    const int qi = qb0 + hf;
    const int tok = 64 * qb0 + r;
    const bool row_valid = tok >= p.row_lo && tok < p.row_hi;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    const uint32_t o_addr = lane_addr + kColO + kOStride * wg;
    const uint32_t l_addr = o_addr + 128;
    const uint32_t* mrow = p.mask + ((size_t)bh * p.Nb + min(qi, p.Nb - 1)) * p.Nw;
    const float sq_row = f.sq[(size_t)bh * p.Nb + min(qi, p.Nb - 1)];
    const float fs_row = sq_row * kScale * kLog2e;   // base-2 score per unit of Q8 . K8, before s_K
    const int n_last = p.N - 64 * (p.Nb - 1);
    const float lg_last = log2f((float)n_last);
    float pivot = -INFINITY;
    bool ok = true;
    bool o1_written = false;
    int t = 0;
    for (;; ++t) {
      const int bsel = t & 1;
      if (!mbar_wait(&sm.dfull[t % kDescRing], (t / kDescRing) & 1, abort) ||
          !mbar_wait(&sm.sfull, t & 1, abort)) {
        ok = false;
        break;
      }
      const TileDesc8 d = sm.desc[t % kDescRing];
      tc_fence_after();
      const bool single = d.kind == kTileSingle;
      o1_written = o1_written || !single;
      const bool pooled = d.kind == kTilePooled;
      const uint32_t s_addr = lane_addr + kColS + 64 * wg;
      const uint32_t p_addr = lane_addr + kColP + 32 * bsel + 16 * wg;
      int lim_own = 64;
      if (!pooled) {
        const bool v = wg ? (!single && ((d.flags >> (2 + hf)) & 1u)) : ((d.flags >> hf) & 1u);
        const int jo = wg ? d.j1 : d.j0;
        lim_own = v ? min(64, p.N - 64 * jo) : 0;
      }
      uint32_t own[64];
      if (lim_own > 0) {
        tmem_ld32_at<0>(s_addr, own);
        tmem_ld32_at<32>(s_addr + 32, own);
        tmem_ld_wait();
        reg_fence(own);
      }
      tc_fence_before();
      mbar_arrive(&sm.sread);
      float* x = reinterpret_cast<float*>(own);
      const float fs = fs_row * (wg ? d.s1 : d.s0);
      float mx = -INFINITY;
      if (lim_own > 0) {
        if (pooled) {
          // base-2 scores in place: scale and log2(n_j) bias; -inf for the row's exact blocks
          const int jb_own = 128 * d.j0 + 64 * wg;
          const int wd0 = 4 * d.j0 + 2 * wg;
          const uint32_t m_own0 = wd0 < p.Nw ? mrow[wd0] : 0xffffffffu;
          const uint32_t m_own1 = wd0 + 1 < p.Nw ? mrow[wd0 + 1] : 0xffffffffu;
          if (jb_own + 64 < p.Nb) {
            // every column a full block other than the last: bias log2 64 throughout
            const uint64_t fs2 = f2(fs, fs), six2 = f2(6.0f, 6.0f);
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
              const float2 v = unf2(fma2(f2(x[c], x[c + 1]), fs2, six2));
              const uint32_t m = (c < 32) ? m_own0 : m_own1;
              x[c] = ((m >> (c & 31)) & 1u) ? -INFINITY : v.x;
              x[c + 1] = ((m >> ((c + 1) & 31)) & 1u) ? -INFINITY : v.y;
            }
          } else {
#pragma unroll
            for (int c = 0; c < 64; ++c) {
              const int j = jb_own + c;
              const float bias = (j == p.Nb - 1) ? lg_last : 6.0f;
              const bool ex = (((c < 32) ? m_own0 : m_own1) >> (c & 31)) & 1u;
              x[c] = (j < p.Nb && !ex) ? fmaf(x[c], fs, bias) : -INFINITY;
            }
          }
        } else if (lim_own < 64) {
#pragma unroll
          for (int c = 0; c < 64; ++c) x[c] = c < lim_own ? x[c] : -INFINITY;
        }
        float mp[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mp[k] = x[k];
#pragma unroll
        for (int c = 8; c < 64; c += 2) mp[(c >> 1) & 7] = max3(mp[(c >> 1) & 7], x[c], x[c + 1]);
        mx = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])), fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
        if (!pooled) mx *= fs;   // exact tiles: raw products, the base-2 scale applied here
      }
      float alpha;
      bool moved;
      const float old_pivot = pivot;
      pivot = pivot_update(pivot, mx, &alpha, &moved);
      uint32_t pk[16];
      if (lim_own > 0) {
        const float c0 = kExpCastOffset - 8.0f * (pivot == -INFINITY ? 0.f : pivot);
        const float f8s = (pooled ? 8.0f : 8.0f * fs) * 0.0078125f, c0s = c0 * 0.0078125f;
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4)
          pk[c4] = expcast_pack4(x[4 * c4], x[4 * c4 + 1], x[4 * c4 + 2], x[4 * c4 + 3], f8s, c0s);
      } else {
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) pk[c4] = 0u;
      }
      // P V of tile t - 1 (and so of t - 2, which read this P buffer) must have completed: O_w and
      // L_w are rescaled below and P_bsel overwritten
      if (t > 0 && !mbar_wait(&sm.pvdone[wg], (t - 1) & 1, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (!(single && wg == 1)) tmem_st16(p_addr, pk);
      // tcgen05.ld / st are warp-collective: the warp rescales if any of its rows needs it
      const bool need = moved && t > 0 && old_pivot != -INFINITY;
      if (__any_sync(0xffffffffu, need)) {
        const float fa = need ? alpha : 1.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t o[64];
          tmem_ld32_at<0>(o_addr + 64 * half, o);
          tmem_ld32_at<32>(o_addr + 64 * half + 32, o);
          tmem_ld_wait();
          reg_fence(o);
#pragma unroll
          for (int e = 0; e < 64; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * fa);
          tmem_st32_at<0>(o_addr + 64 * half, o);
          tmem_st32_at<32>(o_addr + 64 * half + 32, o);
        }
        uint32_t lv = tmem_ld1(l_addr);
        tmem_ld_wait();
        reg_fence1(lv);
        tmem_st1(l_addr, __float_as_uint(__uint_as_float(lv) * fa));
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&sm.pready[wg]);
      if (d.flags & 0x100u) break;
    }
    if (ok && !mbar_wait(&sm.pvdone[wg], t & 1, abort)) ok = false;
    // the row sum of this warpgroup's decoded weights (L_w column 0; L_1 is never written when only
    // 64-key tiles ran, and then its pivot is -inf)
    tc_fence_after();
    float l = 0.f;
    {
      uint32_t lv = tmem_ld1(l_addr);
      tmem_ld_wait();
      reg_fence1(lv);
      if (pivot != -INFINITY) l = __uint_as_float(lv);
    }
    // exchange (pivot, l) with the other warpgroup's thread of this row and merge:
    // o = s_V (O_0 2^(P_0 - M) + O_1 2^(P_1 - M)) / (l_0 2^(P_0 - M) + l_1 2^(P_1 - M)), M = max(P_0, P_1)
    float w_self = 0.f, w_other = 0.f, l_tot = 0.f, m_ref = -INFINITY;
    if (ok) {
      sm.xm[wg][r] = pivot;
      sm.xl[wg][r] = l;
      mbar_arrive(&sm.lbar);
      if (mbar_wait(&sm.lbar, 0, abort)) {
        const float m0 = sm.xm[0][r], m1 = sm.xm[1][r];
        const float l0 = sm.xl[0][r], l1 = sm.xl[1][r];
        const float M = fmaxf(m0, m1);
        const float e0 = M == -INFINITY ? 0.f : pow2i(m0 - M);
        const float e1 = M == -INFINITY ? 0.f : pow2i(m1 - M);
        w_self = wg ? e1 : e0;
        w_other = wg ? e0 : e1;
        l_tot = l0 * e0 + l1 * e1;
        m_ref = M;
      } else {
        ok = false;
      }
    }
    if (!ok) set_timeout(p.status);
    tc_fence_after();
    if (__all_sync(0xffffffffu, ok)) {
      const bool other_written = wg == 1 || o1_written;
      const bool self_written = wg == 0 || o1_written;
      const float sv = f.sv[bh];
      float scale_o = l_tot > 0.f ? sv / l_tot : 0.f;
      float tail_w = 0.f;
      const float* nu = nullptr;
      if (kSol2 && row_valid) {
        const int a = tok / 32;
        const size_t abase = (size_t)bh * p.Na + a;
        const float logz = p.tail_logz[abase];
        if (logz != -INFINITY) {
          // delta_i = (q_i - qbar_a) . mu_a / sqrt(d) with the dequantised query s_Q Q8_i
          const float* mu = p.tail_mu + abase * 128;
          const float* qa = p.qanchor + abase * 128;
          float delta = 0.f;
          const uint32_t q_row = smem_u32(&sm.q[0]) + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll 2
          for (int c16 = 0; c16 < 8; ++c16) {
            const uint32_t addr = q_row + ((((uint32_t)c16) ^ ((uint32_t)r & 7u)) << 4);
            uint32_t w4[4];
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w4[0]), "=r"(w4[1]), "=r"(w4[2]), "=r"(w4[3])
                         : "r"(addr));
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float2 qf = e4m3x2_to_float2((uint16_t)(w4[e >> 1] >> (16 * (e & 1))));
              const int dd = 16 * c16 + 2 * e;
              delta = fmaf(fmaf(qf.x, sq_row, -qa[dd]), mu[dd], delta);
              delta = fmaf(fmaf(qf.y, sq_row, -qa[dd + 1]), mu[dd + 1], delta);
            }
          }
          const float lz2 = (logz + kScale * delta) * kLog2e;   // log2 of Zhat_i
          const float M = fmaxf(m_ref, lz2);
          const float eo = m_ref == -INFINITY ? 0.f : ex2(m_ref - M);
          tail_w = ex2(lz2 - M);
          const float den = l_tot * eo + tail_w;
          scale_o = sv * eo / den;
          tail_w = tail_w / den;
          nu = p.tail_nu + abase * 128 + 64 * wg;
        }
      }
      uint32_t oa[64], ob[64];
      const uint32_t self_addr = lane_addr + kColO + kOStride * wg + 64 * wg;
      const uint32_t other_addr = lane_addr + kColO + kOStride * (1 - wg) + 64 * wg;
      tmem_ld32_at<0>(self_addr, oa);
      tmem_ld32_at<32>(self_addr + 32, oa);
      tmem_ld32_at<0>(other_addr, ob);
      tmem_ld32_at<32>(other_addr + 32, ob);
      tmem_ld_wait();
      reg_fence(oa);
      reg_fence(ob);
      const float ws = (self_written && w_self > 0.f) ? w_self * scale_o : 0.f;
      const float wo = (other_written && w_other > 0.f) ? w_other * scale_o : 0.f;
      if (row_valid) {
        __nv_bfloat16* orow = p.out + ((size_t)((size_t)b * p.N + tok) * p.H + h) * 128 + 64 * wg;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          uint32_t packed[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 8 * c8 + 2 * e;
            float a0 = ws > 0.f ? __uint_as_float(oa[c]) * ws : 0.f;
            float a1 = ws > 0.f ? __uint_as_float(oa[c + 1]) * ws : 0.f;
            if (wo > 0.f) {
              a0 = fmaf(__uint_as_float(ob[c]), wo, a0);
              a1 = fmaf(__uint_as_float(ob[c + 1]), wo, a1);
            }
            if (kSol2 && nu) {
              a0 = fmaf(tail_w, nu[c], a0);
              a1 = fmaf(tail_w, nu[c + 1], a1);
            }
            packed[e] = pack_bf16x2(a0, a1);
          }
          *reinterpret_cast<uint4*>(orow + 8 * c8) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

size_t attn_fwd_fp8_smem_bytes() { return kSmemBytes; }

template <bool kSol2>
static cudaError_t launch_fp8_impl(const CUtensorMap* maps, const FwdParams& p, const Fp8Params& f, int units,
                                   cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_fp8_kernel<kSol2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  attn_fwd_fp8_kernel<kSol2><<<units, 384, kSmemBytes, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], p, f);
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd_fp8(const CUtensorMap* maps, const FwdParams& p, const Fp8Params& f, int units, bool sol2,
                                cudaStream_t st) {
  return sol2 ? launch_fp8_impl<true>(maps, p, f, units, st) : launch_fp8_impl<false>(maps, p, f, units, st);
}

}  // namespace sol
