// Launch interface of the fused attention kernel.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace sol {

struct FwdParams {
  int N, H, Nb, Nw, Na, QT;
  const uint32_t* mask;      // [BH][Nb][Nw]
  int qt_begin, qt_count;    // work units qt_begin .. + qt_count - 1 of each (b, h)
  int unit_blocks;           // query blocks per work unit: 1 (unit u = block u) or 2 (0 also means 2:
                             // unit u = blocks 2u, 2u + 1)
  int row_lo, row_hi;        // token rows [row_lo, row_hi) are written; the others are computed only
  __nv_bfloat16* out;        // [B][N][H][128]
  // split-KV (kv_splits > 1): CTA s of a query tile takes the s-th contiguous share of its key
  // tiles and writes its partial state instead of `out`: part_o [kv_splits][BH][QT * 128][128]
  // (unnormalised O relative to the row's base-2 reference), part_ml [...][2] = (reference, sum)
  int kv_splits;
  float* part_o;
  float* part_ml;
  size_t part_rows_bh;       // BH * QT * 128: rows of one split's partial state
  int* status;               // device status word
  // optional per-CTA timing (nullptr: off): [3 CTA]: start and end of %globaltimer (ns), SM id
  unsigned long long* unit_times;
  // Sol-Attn2 tail (unused by Sol-Attn)
  const float* qanchor;      // [BH][Na][128]
  const float* tail_logz;    // [BH][Na]
  const float* tail_mu;      // [BH][Na][128]
  const float* tail_nu;      // [BH][Na][128]
};

// maps: q, k, v (4-D over BTHD, box 64 channels x 1 head x 64 tokens x 1 batch) and the pooled
// key / value means (3-D over [BH][Nb][128], box 64 channels x 128 blocks x 1).
cudaError_t launch_attn_fwd(const CUtensorMap* maps, const FwdParams& p, int units, bool sol2, cudaStream_t st);
size_t attn_fwd_smem_bytes();

}  // namespace sol
