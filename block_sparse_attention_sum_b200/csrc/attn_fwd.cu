// Fused Sol-Attn forward for sm_100a: exact 64x64 blocks and pooled surrogate tiles through one
// tcgen05 pipeline with one online-softmax state per query row.
//
// Sol-Attn paper (arXiv 2607.24027), section 3.2: "Chunk-wise On-the-Fly Thresholding",
// "Proxy-Score Reuse as Approximate Correction" (token-to-block scores reused for the unselected
// blocks, selected columns masked), "Hardware-Aligned Implementation" (Q_i staged in shared memory,
// one online-softmax state, K/V loaded only for routed blocks; pooled key KC and summed value VC).
// Sol-Attn2 draft, "Routing and complementary approximation" (tail merged in the epilogue).
//
// B200 design (it differs from the paper's nested loop):
//  * A work unit is a 128-row query tile = two adjacent 64-token query blocks, so every tcgen05.mma
//    runs at M = 128.  The unit walks the union of the two blocks' exact sets, two key blocks
//    (128 keys) per tile; columns of a block that is exact for only one half are masked for the
//    other half, whose surrogate then covers that block.
//  * Surrogate tiles: 128 pooled keys Kbar_j (BF16) as the B operand of S = Q K^T and the value
//    means Vbar_j as the B operand of O += P V, with a per-column log-mass bias log2(n_j) and -inf
//    for the columns that are exact for the row's block.  n_j exp(a_j) and exp(a_j) n_j Vbar_j =
//    exp(a_j) Vhat_j are exactly the surrogate's denominator and numerator terms.
//  * Warp roles: warp 0 TMA producer (derives the tile list from the routing bitmask), warp 1 TMEM
//    owner and S = Q K^T issuer, warp 2 O += P V issuer, warps 4-11 two softmax warpgroups (TMEM
//    lane = row; each warpgroup owns 64 of the 128 columns of S, P and O).  S has one buffer in
//    TMEM, released as soon as both warpgroups have loaded it into registers, so the next tile's
//    Q K^T runs while this tile's softmax computes; P (BF16) has its own double buffer; O
//    accumulates in TMEM.
//  * Online softmax in base 2 with a lazily updated reference max: O and l are rescaled only when a
//    row's max grows by more than 2^8, which keeps every probability <= 256.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cfloat>

#include "attn_fwd.cuh"
#include "ptx.cuh"

namespace sol {

namespace {

constexpr int kStages = 3;                     // K / V ring depth
constexpr int kDescRing = 8;                   // tile descriptors in flight (producer <= 3 tiles ahead of
                                               // the MMAs, MMAs <= 2 ahead of the softmax)
constexpr uint32_t kTileBytes = 128 * 64 * 2;  // 128 rows x 64 BF16 columns (one swizzled half, 16 KB)
constexpr uint32_t kBoxBytes = 64 * 64 * 2;    // one 64-row x 64-column BF16 TMA box (8 KB)
// TMEM columns: S (128 x 128 FP32), P double buffer (two x 64 columns, each 128 x 128 BF16 with
// keys 2c, 2c + 1 packed in column c; warpgroup w owns columns 32 w .. 32 w + 31), and one O
// accumulator per softmax warpgroup (each over its half of every tile's keys).
constexpr uint32_t kColS = 0, kColP = 128, kColO = 256;

enum : uint32_t { kTilePair = 0, kTileSingle = 1, kTilePooled = 2 };

struct TileDesc {
  uint32_t kind;
  int j0, j1;       // key blocks (exact tiles) or the pooled chunk index (j0)
  uint32_t flags;   // bit 0/1: j0 exact for half 0/1; bit 2/3: j1 exact for half 0/1; bit 8: last tile
};

struct __align__(1024) FwdSmem {
  __nv_bfloat16 q[2][128 * 64];            // [d half][128 rows x 64], K-major SW128
  __nv_bfloat16 k[kStages][2][128 * 64];   // [stage][d half][128 keys x 64]
  __nv_bfloat16 v[kStages][2][128 * 64];
  TileDesc desc[kDescRing];
  uint64_t kfull[kStages], kempty[kStages], vfull[kStages], vempty[kStages];
  uint64_t dfull[kDescRing];
  uint64_t qfull, sfull, sread, pready[2], pvdone[2], mmadone, mmadone2;
  uint64_t lbar;            // softmax warpgroups: (max, sum) exchange before the epilogue merge
  float xm[2][128], xl[2][128];   // [warpgroup][row] running max and row sum, for the epilogue merge
  uint32_t tmem_base;
  int abort;
  int tile_lo, tile_hi;     // this CTA's share [tile_lo, tile_hi) of the unit's tile list
  unsigned long long t_start;   // %globaltimer at the CTA's start (per-CTA timing only)
};

// The dynamic shared-memory window starts 1024-byte aligned on sm_100 (checked at run time: a
// misaligned base is reported through the status word and the CTA exits without touching memory).
constexpr size_t kSmemBytes = sizeof(FwdSmem);
static_assert(kSmemBytes <= 232448, "shared memory budget");

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

// Packed FP32 pairs (sm_100 f32x2 arithmetic).
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

__device__ __forceinline__ void set_timeout(int* status) { atomicExch(status, kDevTimeout); }

// Debug builds (-DSOL_ATTN_DEBUG_BOUNDS) check every TMA tile coordinate against the tensor it
// reads; a failed check records kDevBounds in the status word and the copy is skipped (its consumer
// then runs out its bounded wait).  Release builds compile the checks away.
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
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kp,
                    const __grid_constant__ CUtensorMap tm_vp, const FwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_u32(smem_raw) & 1023u) {   // uniform across the CTA
    if (tid == 0) atomicExch(p.status, kDevMisaligned);
    return;
  }
  FwdSmem& sm = *reinterpret_cast<FwdSmem*>(smem_raw);
  volatile int* abort = &sm.abort;

  const int unit = (int)blockIdx.x / p.kv_splits, split = (int)blockIdx.x % p.kv_splits;
  const int bh = unit / p.qt_count, qt = p.qt_begin + unit % p.qt_count;
  const int b = bh / p.H, h = bh % p.H;
  const bool one_block = p.unit_blocks == 1;   // m_tile 64: one query block, rows 64..127 idle
  const int qb0 = one_block ? qt : 2 * qt;
  const bool has_hi = !one_block && qb0 + 1 < p.Nb;

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
    if (p.unit_times) sm.t_start = globaltimer();
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 2) {
    // the unit's tile count (exact pairs over the union of its two rows, then surrogate chunks),
    // split into kv_splits contiguous shares; one share for the whole list without split-KV
    int lo = 0, hi = 0x7fffffff;
    if (p.kv_splits > 1) {
      const uint32_t* row0 = p.mask + ((size_t)bh * p.Nb + qb0) * p.Nw;
      const uint32_t* row1 = row0 + p.Nw;
      int uni = 0, pooled_tiles = 0;
      for (int wd = lane; wd < p.Nw; wd += 32) {
        const uint32_t a = row0[wd], c = has_hi ? row1[wd] : 0u;
        uni += __popc(a | c);
      }
      if (!kSol2) {
        for (int ch = lane; ch < (p.Nb + 127) / 128; ch += 32) {
          bool any = false;
          for (int e = 0; e < 4; ++e) {
            const int wd = 4 * ch + e;
            if (wd >= p.Nw) break;
            const int nvalid = min(32, p.Nb - 32 * wd);
            const uint32_t valid = nvalid >= 32 ? 0xffffffffu : ((1u << nvalid) - 1u);
            if ((~row0[wd] & valid) || (has_hi && (~row1[wd] & valid))) any = true;
          }
          pooled_tiles += any ? 1 : 0;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        uni += __shfl_xor_sync(0xffffffffu, uni, o);
        pooled_tiles += __shfl_xor_sync(0xffffffffu, pooled_tiles, o);
      }
      const int total = (uni + 1) / 2 + pooled_tiles;
      lo = (int)((long long)total * split / p.kv_splits);
      hi = (int)((long long)total * (split + 1) / p.kv_splits);
    }
    if (lane == 0) {
      sm.tile_lo = lo;
      sm.tile_hi = hi;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const bool empty_share = sm.tile_lo >= sm.tile_hi;   // split-KV: no key tile for this CTA

  if (warp == 0) {
    // ----------------------------------------------------------------------------------- producer
    if (lane == 0 && !empty_share) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      if (!kSol2) {
        tma_prefetch_desc(&tm_kp);
        tma_prefetch_desc(&tm_vp);
      }
      mbar_arrive_expect_tx(&sm.qfull, 4 * kBoxBytes);
      if (tile_ok(1u, qb0, 0, p.Nb, p.status))
      for (int hf = 0; hf < 2; ++hf)
        for (int dh = 0; dh < 2; ++dh)
          tma_load_4d(&sm.q[dh][hf * 64 * 64], &tm_q, &sm.qfull, 64 * dh, h, 64 * (qb0 + hf), b);

      const uint32_t* row0 = p.mask + ((size_t)bh * p.Nb + qb0) * p.Nw;
      const uint32_t* row1 = row0 + p.Nw;
      int t = 0;
      bool ok = true;
      TileDesc prev;
      bool have_prev = false;
      auto issue = [&](TileDesc d) {
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
        const uint32_t bytes = pooled ? 2 * kTileBytes : 2 * kBoxBytes * nblk;
        mbar_arrive_expect_tx(&sm.kfull[s], bytes);
        if (!tile_ok(d.kind, d.j0, d.j1, p.Nb, p.status)) {
        } else if (pooled) {
          for (int dh = 0; dh < 2; ++dh) tma_load_3d(&sm.k[s][dh][0], &tm_kp, &sm.kfull[s], 64 * dh, 128 * d.j0, bh);
        } else {
          for (int slot = 0; slot < nblk; ++slot)
            for (int dh = 0; dh < 2; ++dh)
              tma_load_4d(&sm.k[s][dh][slot * 64 * 64], &tm_k, &sm.kfull[s], 64 * dh, h, 64 * (slot ? d.j1 : d.j0),
                          b);
        }
        ++t;
      };
      int g = 0;   // index of the next tile in the unit's list (split-KV keeps [tile_lo, tile_hi))
      const int g_lo = sm.tile_lo, g_hi = sm.tile_hi;
      auto push = [&](TileDesc d) {
        const int gi = g++;
        if (gi < g_lo || gi >= g_hi) return;
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
            push(TileDesc{kTilePair, pend, j, pend_fl | (fl << 2)});
            pend = -1;
          }
        }
      }
      if (pend >= 0 && ok) push(TileDesc{kTileSingle, pend, pend, pend_fl});
      if (!kSol2) {
        // surrogate tiles: 128 pooled keys each; skip chunks that are exact for both rows
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
          if (any) push(TileDesc{kTilePooled, ch, ch, 0});
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
    if (lane == 0 && !empty_share) {
      bool ok = mbar_wait(&sm.qfull, 0, abort);
      const uint32_t q_base = smem_u32(&sm.q[0][0]);
      for (int t = 0; ok; ++t) {
        const int s = t % kStages;
        if (!mbar_wait(&sm.kfull[s], (t / kStages) & 1, abort)) {
          ok = false;
          break;
        }
        const TileDesc d = sm.desc[t % kDescRing];
        // S still holds tile t - 1 until both softmax warpgroups have loaded it
        if (t >= 1 && !mbar_wait(&sm.sread, (t - 1) & 1, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int n = d.kind == kTileSingle ? 64 : 128;
        const uint32_t idesc = idesc_bf16(128, n, false, false);
        const uint32_t k_base = smem_u32(&sm.k[s][0][0]);
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kTileBytes + (kk & 3) * 32;
          umma_ss(tmem + kColS, sdesc_sw128(q_base + off, 16, 1024),
                  sdesc_sw128(k_base + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
        }
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
    // ------------------------------------------------------------------------------ O += P V issuer
    // One product per softmax warpgroup and tile: O_w += P_w V_w over the warpgroup's 64 keys, issued
    // as soon as that warpgroup's P is in TMEM.  A separate thread from the Q K^T issuer, so neither
    // queues behind the other in program order.
    if (lane == 0 && !empty_share) {
      bool ok = true;
      bool b_started = false;
      for (int u = 0; ok; ++u) {
        const int s = u % kStages;
        const int bsel = u & 1;
        if (!mbar_wait(&sm.dfull[u % kDescRing], (u / kDescRing) & 1, abort) ||
            !mbar_wait(&sm.vfull[s], (u / kStages) & 1, abort)) {
          ok = false;
          break;
        }
        const TileDesc d = sm.desc[u % kDescRing];
        const uint32_t idesc = idesc_bf16(128, 128, false, true);
        const uint32_t v_base = smem_u32(&sm.v[s][0][0]);
        for (int w = 0; w < 2 && ok; ++w) {
          if (!mbar_wait(&sm.pready[w], u & 1, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const bool skip = (w == 1 && d.kind == kTileSingle);   // no keys in the second half
          if (!skip) {
            const uint32_t p_col = tmem + kColP + 64 * bsel + 32 * w;   // P_w: 64 keys in 32 columns
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t bd = sdesc_sw128(v_base + (4 * w + kk) * 2048, kTileBytes, 1024);
              const bool acc = w == 0 ? (u > 0 || kk > 0) : (b_started || kk > 0);
              umma_ts(tmem + kColO + 128 * w, p_col + 8 * kk, bd, idesc, acc ? 1u : 0u);
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
    // Loads V tiles in the order the K producer published them, so that K tiles (needed first, by
    // Q K^T) never wait behind the release of a V stage.
    if (lane == 0 && !empty_share) {
      bool ok = true;
      int u = 0;
      for (;; ++u) {
        const int s = u % kStages;
        if (!mbar_wait(&sm.dfull[u % kDescRing], (u / kDescRing) & 1, abort) ||
            (u >= kStages && !mbar_wait(&sm.vempty[s], ((u / kStages) - 1) & 1, abort))) {
          ok = false;
          break;
        }
        const TileDesc d = sm.desc[u % kDescRing];
        const bool pooled = d.kind == kTilePooled;
        const int nblk = d.kind == kTilePair ? 2 : 1;
        mbar_arrive_expect_tx(&sm.vfull[s], pooled ? 2 * kTileBytes : 2 * kBoxBytes * nblk);
        if (!tile_ok(d.kind, d.j0, d.j1, p.Nb, p.status)) {
        } else if (pooled) {
          for (int dh = 0; dh < 2; ++dh) tma_load_3d(&sm.v[s][dh][0], &tm_vp, &sm.vfull[s], 64 * dh, 128 * d.j0, bh);
        } else {
          for (int slot = 0; slot < nblk; ++slot)
            for (int dh = 0; dh < 2; ++dh)
              tma_load_4d(&sm.v[s][dh][slot * 64 * 64], &tm_v, &sm.vfull[s], 64 * dh, h, 64 * (slot ? d.j1 : d.j0),
                          b);
        }
        if (d.flags & 0x100u) {
          ++u;
          break;
        }
      }
      if (!ok) set_timeout(p.status);
      // never leave the CTA with bulk copies in flight
      for (int w = max(0, u - kStages); w < u; ++w) mbar_wait(&sm.vfull[w % kStages], (w / kStages) & 1, abort);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // --------------------------------------------------------------- softmax / correction / epilogue
    // Two warpgroups share the 128 rows (TMEM lane = row); warpgroup wg owns columns 64 wg .. 64 wg + 63
    // of every tile and keeps its own online-softmax state (m, l) and its own O accumulator over
    // those keys.  The two partial results of a row are merged exactly in the epilogue, so the
    // warpgroups never wait for each other inside the tile loop.
    const int wg = (warp - 4) >> 2;
    const int r = ((warp & 3) << 5) | lane;   // query row within the tile == TMEM lane
    const int hf = r >> 6;
    const int qi = qb0 + hf;
    const int tok = 64 * qb0 + r;
    const bool row_valid = (r < 64 || has_hi) && tok >= p.row_lo && tok < p.row_hi;
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    const uint32_t o_addr = lane_addr + kColO + 128 * wg;
    const uint32_t* mrow = p.mask + ((size_t)bh * p.Nb + min(qi, p.Nb - 1)) * p.Nw;
    const float sc = kScale * kLog2e;
    const int n_last = p.N - 64 * (p.Nb - 1);
    const float lg_last = log2f((float)n_last);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    if (empty_share) {
      if (wg == 0 && row_valid) {
        const size_t prow = (size_t)(blockIdx.x % p.kv_splits) * p.part_rows_bh + (size_t)bh * p.QT * 128 + tok;
        p.part_ml[2 * prow] = -INFINITY;   // no key in this share: weight 0 in the combine
        p.part_ml[2 * prow + 1] = 0.f;
      }
    } else {
    bool o1_written = false;   // O_1 receives a product for every tile with a second 64-key half
    int t = 0;
    for (;; ++t) {
      const int bsel = t & 1;
      if (!mbar_wait(&sm.dfull[t % kDescRing], (t / kDescRing) & 1, abort) ||
          !mbar_wait(&sm.sfull, t & 1, abort)) {
        ok = false;
        break;
      }
      const TileDesc d = sm.desc[t % kDescRing];
      tc_fence_after();
      const bool single = d.kind == kTileSingle;
      o1_written = o1_written || !single;
      const bool pooled = d.kind == kTilePooled;
      const uint32_t s_addr = lane_addr + kColS + 64 * wg;
      const uint32_t p_addr = lane_addr + kColP + 64 * bsel + 32 * wg;
      // columns of this warpgroup's half that are valid for its row (warp-uniform)
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
      // S is in registers: the next tile's Q K^T may overwrite it
      tc_fence_before();
      mbar_arrive(&sm.sread);
      // x: this warpgroup's 64 columns in place over the raw scores.  Exact tiles keep raw scores
      // (the base-2 scale is folded into the exponent), pooled tiles carry scale and log2(n_j) bias.
      float* x = reinterpret_cast<float*>(own);
      float mx = -INFINITY;
      if (lim_own > 0) {
        if (pooled) {
          const int jb_own = 128 * d.j0 + 64 * wg;
          const int wd0 = 4 * d.j0 + 2 * wg;
          const uint32_t m_own0 = wd0 < p.Nw ? mrow[wd0] : 0xffffffffu;
          const uint32_t m_own1 = wd0 + 1 < p.Nw ? mrow[wd0 + 1] : 0xffffffffu;
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const int j = jb_own + c;
            const float bias = (j == p.Nb - 1) ? lg_last : 6.0f;
            const bool ex = (((c < 32) ? m_own0 : m_own1) >> (c & 31)) & 1u;
            x[c] = (j < p.Nb && !ex) ? fmaf(x[c], sc, bias) : -INFINITY;
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
        if (!pooled) mx *= sc;   // exact tiles: raw scores, base-2 scale applied here
      }
      const float m_new = fmaxf(m_ref, mx);
      const bool upd = m_new > m_ref + 8.0f;
      const float m_use = upd ? m_new : m_ref;
      const float m_sub = m_use == -INFINITY ? 0.f : m_use;
      const float alpha = upd ? ex2(m_ref - m_sub) : 1.f;
      uint64_t rs2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
      uint32_t pk[32];
      if (lim_own > 0) {
        const float fs = pooled ? 1.f : sc;
        const uint64_t fs2 = f2(fs, fs), nm2 = f2(-m_sub, -m_sub);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float2 y = unf2(fma2(f2(x[2 * c], x[2 * c + 1]), fs2, nm2));
          const float2 pp = make_float2(ex2(y.x), ex2(y.y));
          rs2[c & 1] = add2(rs2[c & 1], f2(pp.x, pp.y));
          pk[c] = pack_bf16x2(pp.x, pp.y);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      }
      const float2 rsa = unf2(add2(rs2[0], rs2[1]));
      l = l * alpha + (rsa.x + rsa.y);
      // P V of tile t - 1 (and so of t - 2, which read this P buffer) must have completed: O_w is
      // rescaled below and P_bsel overwritten
      if (t > 0 && !mbar_wait(&sm.pvdone[wg], (t - 1) & 1, abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (!(single && wg == 1)) tmem_st32(p_addr, pk);
      // tcgen05.ld / st are warp-collective: the warp rescales if any of its rows needs it
      const bool need = upd && t > 0 && m_ref != -INFINITY;
      if (__any_sync(0xffffffffu, need)) {
        const float f = need ? alpha : 1.f;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t o[64];
          tmem_ld32_at<0>(o_addr + 64 * half, o);
          tmem_ld32_at<32>(o_addr + 64 * half + 32, o);
          tmem_ld_wait();
          reg_fence(o);
#pragma unroll
          for (int e = 0; e < 64; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
          tmem_st32_at<0>(o_addr + 64 * half, o);
          tmem_st32_at<32>(o_addr + 64 * half + 32, o);
        }
      }
      m_ref = m_use;
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&sm.pready[wg]);
      if (d.flags & 0x100u) break;
    }
    if (ok && !mbar_wait(&sm.pvdone[wg], t & 1, abort)) ok = false;
    // exchange (m, l) with the other warpgroup's thread of this row, then merge the two halves:
    // o = (O_0 2^(m_0 - M) + O_1 2^(m_1 - M)) / (l_0 2^(m_0 - M) + l_1 2^(m_1 - M)), M = max(m_0, m_1)
    float w_self = 0.f, w_other = 0.f, l_tot = 1.f;
    if (ok) {
      sm.xm[wg][r] = m_ref;
      sm.xl[wg][r] = l;
      mbar_arrive(&sm.lbar);
      if (mbar_wait(&sm.lbar, 0, abort)) {
        const float m0 = sm.xm[0][r], m1 = sm.xm[1][r];
        const float l0 = sm.xl[0][r], l1 = sm.xl[1][r];
        const float M = fmaxf(m0, m1);
        const float e0 = m0 == -INFINITY ? 0.f : ex2(m0 - M);
        const float e1 = m1 == -INFINITY ? 0.f : ex2(m1 - M);
        w_self = wg ? e1 : e0;
        w_other = wg ? e0 : e1;
        l_tot = l0 * e0 + l1 * e1;
        m_ref = M;   // the merged row's reference (base 2)
      } else {
        ok = false;
      }
    }
    if (!ok) set_timeout(p.status);
    tc_fence_after();
    if (__all_sync(0xffffffffu, ok)) {
      // epilogue: this warpgroup writes output columns 64 wg .. 64 wg + 63 from both accumulators
      const bool other_written = wg == 1 || o1_written;   // O_1 exists unless only 64-key tiles ran
      const bool self_written = wg == 0 || o1_written;
      float scale_o = 1.f / l_tot;
      float tail_w = 0.f;
      const float* nu = nullptr;
      if (kSol2) {
        // the warp's 32 rows share one anchor: the warp loads mu_a and this warpgroup's half of
        // nu_a once (coalesced) into the idle K ring (every product is complete here) and reduces
        // qbar_a . mu_a; each lane then reads them as shared-memory broadcasts, and
        // delta_i = (q_i . mu_a - qbar_a . mu_a) / sqrt(d)
        const int a = min(2 * qb0 + (warp & 3), p.Na - 1);
        const size_t abase = (size_t)bh * p.Na + a;
        const float logz = p.tail_logz[abase];
        if (logz != -INFINITY) {   // warp-uniform
          float* sc_mu = reinterpret_cast<float*>(&sm.k[0][0][0]) + (warp - 4) * 192;
          float* sc_nu = sc_mu + 128;
          const float4 m4 = reinterpret_cast<const float4*>(p.tail_mu + abase * 128)[lane];
          const float4 q4 = reinterpret_cast<const float4*>(p.qanchor + abase * 128)[lane];
          float qm = fmaf(m4.x, q4.x, fmaf(m4.y, q4.y, fmaf(m4.z, q4.z, m4.w * q4.w)));
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) qm += __shfl_xor_sync(0xffffffffu, qm, o);
          reinterpret_cast<float4*>(sc_mu)[lane] = m4;
          if (lane < 16)
            reinterpret_cast<float4*>(sc_nu)[lane] = reinterpret_cast<const float4*>(p.tail_nu + abase * 128 + 64 * wg)[lane];
          __syncwarp();
          if (row_valid) {
            float dot = 0.f;
            const uint32_t q_row = smem_u32(&sm.q[0][0]) + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll 4
            for (int c8 = 0; c8 < 16; ++c8) {
              const uint32_t addr = q_row + (c8 >> 3) * kTileBytes + ((((uint32_t)c8 & 7u) ^ ((uint32_t)r & 7u)) << 4);
              uint32_t w4[4];
              asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(w4[0]), "=r"(w4[1]), "=r"(w4[2]), "=r"(w4[3])
                           : "r"(addr));
              const float4 ma = reinterpret_cast<const float4*>(sc_mu)[2 * c8];
              const float4 mb = reinterpret_cast<const float4*>(sc_mu)[2 * c8 + 1];
              const float mu8[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
                dot = fmaf(f.x, mu8[2 * e], dot);
                dot = fmaf(f.y, mu8[2 * e + 1], dot);
              }
            }
            const float lz2 = (logz + kScale * (dot - qm)) * kLog2e;  // log2 of Zhat_i
            const float M = fmaxf(m_ref, lz2);
            const float eo = ex2(m_ref - M);
            tail_w = ex2(lz2 - M);
            const float den = l_tot * eo + tail_w;
            scale_o = eo / den;
            tail_w = tail_w / den;
            nu = sc_nu;
          }
        }
      }
      // O_self columns 64 wg.. and O_other columns 64 wg.. (the other accumulator's same columns)
      uint32_t oa[64], ob[64];
      const uint32_t self_addr = lane_addr + kColO + 128 * wg + 64 * wg;
      const uint32_t other_addr = lane_addr + kColO + 128 * (1 - wg) + 64 * wg;
      tmem_ld32_at<0>(self_addr, oa);
      tmem_ld32_at<32>(self_addr + 32, oa);
      tmem_ld32_at<0>(other_addr, ob);
      tmem_ld32_at<32>(other_addr + 32, ob);
      tmem_ld_wait();
      reg_fence(oa);
      reg_fence(ob);
      const float ws = (self_written && w_self > 0.f) ? w_self * scale_o : 0.f;
      const float wo = (other_written && w_other > 0.f) ? w_other * scale_o : 0.f;
      if (p.kv_splits > 1) {
        // split-KV: the partial state of this share (O relative to the merged reference m_ref)
        if (row_valid) {
          const size_t prow = (size_t)(blockIdx.x % p.kv_splits) * p.part_rows_bh + (size_t)bh * p.QT * 128 + tok;
          float* dst = p.part_o + prow * 128 + 64 * wg;
#pragma unroll
          for (int c = 0; c < 64; c += 4) {
            float o4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float a = w_self > 0.f ? __uint_as_float(oa[c + e]) * w_self : 0.f;
              if (w_other > 0.f) a = fmaf(__uint_as_float(ob[c + e]), w_other, a);
              o4[e] = a;
            }
            *reinterpret_cast<float4*>(dst + c) = make_float4(o4[0], o4[1], o4[2], o4[3]);
          }
          if (wg == 0) {
            p.part_ml[2 * prow] = m_ref;
            p.part_ml[2 * prow + 1] = l_tot;
          }
        }
      } else if (row_valid) {
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
    }   // non-empty share
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (p.unit_times && tid == 0) {
    unsigned smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    unsigned long long* u = p.unit_times + 3 * (size_t)blockIdx.x;
    u[0] = sm.t_start;
    u[1] = globaltimer();
    u[2] = smid;
  }
}

size_t attn_fwd_smem_bytes() { return kSmemBytes; }

template <bool kSol2>
static cudaError_t launch_impl(const CUtensorMap* maps, const FwdParams& p, int units, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<kSol2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  attn_fwd_kernel<kSol2><<<units, 384, kSmemBytes, st>>>(maps[0], maps[1], maps[2], maps[3], maps[4], p);
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd(const CUtensorMap* maps, const FwdParams& p, int units, bool sol2, cudaStream_t st) {
  return sol2 ? launch_impl<true>(maps, p, units, st) : launch_impl<false>(maps, p, units, st);
}

}  // namespace sol
