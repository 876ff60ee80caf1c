// Launch interface of the fused FP8 (E4M3) + ExpCast attention kernel.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "attn_fwd.cuh"

namespace sol {

// E4M3 scales (quant_fp8.cu); the other arguments are those of the BF16 kernel (FwdParams, with
// kv_splits = 1: the FP8 kernel writes `out` directly).
struct Fp8Params {
  const float* sq;      // [BH][Nb]       per 64-token query block
  const float* sk;      // [BH][Nb]       per 64-token key block
  const float* skbar;   // [BH][gk]       per 64 compressed keys
  const float* sv;      // [BH]           per head
  int gk;               // scale groups of the compressed keys per head (Nbp / 64)
};

// maps: q8, k8, v8 (4-D over BTHD bytes, box 128 channels x 1 head x 64 tokens x 1 batch) and the
// E4M3 compressed keys / values (3-D over [BH][Nbp][128] bytes, box 128 channels x 128 rows x 1);
// all with the 128-byte swizzle.
cudaError_t launch_attn_fwd_fp8(const CUtensorMap* maps, const FwdParams& p, const Fp8Params& f, int units, bool sol2,
                                cudaStream_t st);
size_t attn_fwd_fp8_smem_bytes();

}  // namespace sol
