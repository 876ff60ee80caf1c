// Shapes, workspace layout and kernel declarations shared by the host launcher and the kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace sol {

constexpr int kHeadDim = 128;   // head dimension (fixed by the operator's contract)
constexpr int kBlock = 64;      // query / key block size (64 x 64 physical blocks)
constexpr int kAnchor = 32;     // Sol-Attn2 query anchor size
constexpr float kScale = 0.088388347648318440550f;        // 1 / sqrt(128)
constexpr float kLog2e = 1.4426950408889634074f;

struct Shape {
  int B, N, H;
  int Nb;   // key / query blocks
  int Nw;   // 32-bit words per bitmask row
  int Na;   // Sol-Attn2 anchors
  int BH;
  int QT;   // 128-row query tiles (pairs of query blocks)
};

inline Shape make_shape(int B, int N, int H) {
  Shape s;
  s.B = B;
  s.N = N;
  s.H = H;
  s.Nb = (N + kBlock - 1) / kBlock;
  s.Nw = (s.Nb + 31) / 32;
  s.Na = (N + kAnchor - 1) / kAnchor;
  s.BH = B * H;
  s.QT = (s.Nb + 1) / 2;
  return s;
}

// Device buffers of one call (all inside the library workspace).
struct Work {
  float* qbar;            // [BH][Nb][128]  block means of Q
  float* kbar;            // [BH][Nb][128]  block means of K
  __nv_bfloat16* kbar_h;  // [BH][Nb][128]  BF16 copy of kbar (surrogate MMA operand)
  __nv_bfloat16* vbar_h;  // [BH][Nb][128]  BF16 block means of V (surrogate MMA operand)
  __nv_bfloat16* qbar_hi; // [BH][Nb][128]  bf16(qbar)            } two-term BF16 splits of the
  __nv_bfloat16* qbar_lo; // [BH][Nb][128]  bf16(qbar - qbar_hi)  } means for the routing product
  __nv_bfloat16* kbar_lo; // [BH][Nb][128]  bf16(kbar - kbar_h)   } (kbar_h is the hi part of kbar)
  float* kcov;            // [BH][128][128] centred covariance of the key-block means
  float* gram_partial;    // [BH][8][128][128] partial Gram sums over ranges of key blocks
  double* kmean;          // [BH][128]      mean of the key-block means
  float* thresh;          // [BH][Nb]       tau_i
  uint32_t* mask;         // [BH][Nb][Nw]   exact-block bitmask
  int* rowcount;          // [BH][Nb]       exact blocks per query-block row
  unsigned long long* stats;  // [0] exact pairs, [1] min row, [2] max row (as unsigned)
  // Sol-Attn2
  float* qanchor;         // [BH][Na][128]  anchor means of Q
  __nv_bfloat16* qanchor_h;  // [BH][Na][128] BF16 copy (tail MMA operand)
  float* qdir;            // [BH][128]      mean query (the grouping direction)
  __nv_bfloat16* gk_h;    // [BH][Nb][2][128] group key means (BF16, tail MMA operand)
  __nv_bfloat16* gv_h;    // [BH][Nb][2][128] group value means (BF16, tail MMA operand)
  float* glog2n;          // [BH][Gp]       log2 of the group sizes, -inf for empty groups and
                          //                the padding up to Gp = 2 Nb rounded up to 128
  float* tail_logz;       // [BH][Na]       log Z_a (-inf for an empty tail)
  float* tail_mu;         // [BH][Na][128]
  float* tail_nu;         // [BH][Na][128]
};

// Sets the calling thread's message returned by sol_attn_last_error() (api.cu).
void set_last_error(const char* msg);

struct Fp8Work;

// Prep kernels (summary.cu).  With f8, the summary pass also writes the E4M3 codes of Q and K with
// their block scales and folds max |V| of every block into the head's maximum (f8->vmax, cleared
// before the call).
void launch_summary(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, const Shape& s,
                    const Work& w, bool anchors, cudaStream_t st, const Fp8Work* f8 = nullptr);
void launch_kstats(const Shape& s, const Work& w, cudaStream_t st);
void launch_thresh(const Shape& s, const Work& w, float tau, bool diag, cudaStream_t st);
// Routing on the tensor cores (route_tc.cu); maps = qbar_hi, qbar_lo, kbar_h, kbar_lo (BF16, 3-D,
// box 64 x 128 x 1, 128-byte swizzle).
// Exact key-block ranges forced by the sinks: inclusive block intervals [b0[e], b1[e]].
constexpr int kMaxSinkRanges = 5;   // the sink_start / sink_tokens range and up to 4 extra ranges
struct SinkSet {
  int n;
  int b0[kMaxSinkRanges], b1[kMaxSinkRanges];
};
// Split-KV combine (splitkv.cu): merges the kv_splits partial states of every query row into out.
void launch_splitkv_combine(const Shape& s, int splits, const float* part_o, const float* part_ml,
                            __nv_bfloat16* out, int row_lo, int row_hi, cudaStream_t st);
cudaError_t launch_route_tc(const void* maps, const Shape& s, const Work& w, const SinkSet& sinks, int* status,
                            cudaStream_t st);
void launch_expand_mask(const Shape& s, const Work& w, unsigned char* mask_out, cudaStream_t st);
// Sets every valid bit of the bitmask rows of query blocks qb_lo .. qb_hi (all heads).
void launch_dense_mask(const Shape& s, const Work& w, int qb_lo, int qb_hi, cudaStream_t st);

// Sol-Attn2 summaries (sol2_tail.cu), in place of launch_summary: query and anchor means, the mean
// query, then key means and the two key groups of every block (three launches).
void launch_sol2_summaries(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, const Shape& s,
                           const Work& w, cudaStream_t st, const Fp8Work* f8 = nullptr);
// Sol-Attn2 tail statistics on the tensor cores (sol2_tail_tc.cu); maps = anchor means, group key
// means, group value means (BF16, 3-D, box 64 x 128 x 1, 128-byte swizzle).
cudaError_t launch_tail_tc(const void* maps, const Shape& s, const Work& w, int* status, cudaStream_t st);
__host__ __device__ inline int tail_groups_padded(const Shape& s) { return (2 * s.Nb + 127) / 128 * 128; }

// FP8 path (quant_fp8.cu, attn_fwd_fp8.cu): E4M3 operands and their scales.
struct Fp8Work {
  uint8_t* q8;            // [B][N][H][128]  E4M3 Q, one scale per (b, h, 64-token block)
  uint8_t* k8;            // [B][N][H][128]  E4M3 K, same
  uint8_t* v8;            // [B][N][H][128]  E4M3 V, one scale per (b, h)
  uint8_t* kbar8;         // [BH][Nbp][128]  E4M3 compressed keys (block means), one scale per 64 rows
  uint8_t* vbar8;         // [BH][Nbp][128]  E4M3 value means, the head's V scale
  float* sq;              // [BH][Nb]
  float* sk;              // [BH][Nb]
  float* skbar;           // [BH][Nbp / 64]
  float* sv;              // [BH]
  unsigned int* vmax;     // [BH] max |V| of the head (float bits)
};
// Rows of the compressed-key arrays: Nb rounded up to whole 128-row surrogate chunks.
__host__ __device__ inline int fp8_rows_padded(const Shape& s) { return (s.Nb + 127) / 128 * 128; }
// V (head scale) and the compressed keys / values; Q and K come from the summary pass (f8 there).
void launch_quant_fp8(const __nv_bfloat16* v, const Shape& s, const Work& w, const Fp8Work& f, cudaStream_t st);

}  // namespace sol
