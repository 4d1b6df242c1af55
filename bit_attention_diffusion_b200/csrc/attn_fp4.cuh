// attn_fp4.cuh - launch parameters of the fused attention kernel of the
// NVFP4-residual variant (QK^T in FP8, or in NVFP4 for the full 4-bit path).
#pragma once
#include <cstdint>
#include <cuda.h>

namespace vc {

struct AttnFp4Params {
  int N, Nb, Npad, nch32, R, Rpad;
  float kappa;                // 8 * log2(e) * softmax_scale
  const float *sq, *sk;       // [BH][Nb] block scales of Q8 and K8 (QK4: power-of-two global scales of Q4, K4')
  const float *vscale;        // [BH][128] power-of-two global scales g of the NVFP4 residual
  const uint8_t *v4img;       // [BH][Nb] NVFP4 tile images (V4_TILE_BYTES each)
  const uint8_t *qimg, *kimg; // QK4: [BH][Nb] NVFP4 tile images of Q and K' (rows = tokens); else null
  const int32_t *rep_idx;     // [BH][R] permuted positions of repaired tokens
  const uint8_t *k8;          // [BH][Npad][128] (8-bit QK^T: the repair gathers rows from it)
  uint16_t *O;                // [BH][N][128] bf16 output
  uint32_t *status;           // device status word
};

// Grid ceil(Nb/2) x B*H: CTA x takes query tiles 2x and 2x+1. QK^T from the E4M3 tiles (tmQ, tmK).
__global__ void k_vc_attn_fwd4(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                               const __grid_constant__ CUtensorMap tmMu, const __grid_constant__ CUtensorMap tmDT,
                               const AttnFp4Params p);
// The full 4-bit path: QK^T from the NVFP4 images of Q and K' (tmQ, tmK unused).
__global__ void k_vc_attn_fwd44(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                                const __grid_constant__ CUtensorMap tmMu, const __grid_constant__ CUtensorMap tmDT,
                                const AttnFp4Params p);
uint32_t attn_fp4_smem_bytes(bool qk4);

}  // namespace vc
