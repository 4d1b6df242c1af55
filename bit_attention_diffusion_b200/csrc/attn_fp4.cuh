// attn_fp4.cuh - launch parameters of the fused attention kernel of the
// NVFP4-residual variant.
#pragma once
#include <cstdint>
#include <cuda.h>

namespace vc {

struct AttnFp4Params {
  int N, Nb, Npad, nch32, R, Rpad;
  float kappa;                // 8 * log2(e) * softmax_scale
  const float *sq, *sk;       // [BH][Nb] block scales of Q8 and K8
  const float *vscale;        // [BH][128] power-of-two global scales g of the NVFP4 residual
  const uint8_t *v4img;       // [BH][Nb] NVFP4 tile images (V4_TILE_BYTES each)
  const int32_t *rep_idx;     // [BH][R] permuted positions of repaired tokens
  const uint8_t *k8;          // [BH][Npad][128] (repair gathers rows from it)
  uint16_t *O;                // [BH][N][128] bf16 output
  uint32_t *status;           // device status word
};

__global__ void k_vc_attn_fwd4(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                               const __grid_constant__ CUtensorMap tmMu, const __grid_constant__ CUtensorMap tmDT,
                               const AttnFp4Params p);
uint32_t attn_fp4_smem_bytes();

}  // namespace vc
