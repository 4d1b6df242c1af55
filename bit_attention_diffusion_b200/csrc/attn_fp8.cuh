// attn_fp8.cuh - launch parameters of the fused FP8 attention kernel.
#pragma once
#include <cstdint>
#include <cuda.h>

namespace vc {

struct AttnFp8Params {
  int N, Nb, Npad, nch32, R, Rpad, C;
  float kappa;                // 8 * log2(e) * softmax_scale
  const float *sq, *sk;       // [BH][Nb] block scales of Q8 and K8
  const float *vscale;        // [BH][128] power-of-two V residual scales
  const int32_t *rep_idx;     // [BH][R] permuted positions of repaired tokens
  const uint8_t *k8;          // [BH][Npad][128] (repair gathers rows from it)
  uint16_t *O;                // [BH][N][128] bf16 output
  uint32_t *status;           // device status word
};

// Grid ceil(Nb/2) x B*H: CTA x takes query tiles 2x and 2x+1.
__global__ void k_vc_attn_fwd(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmMu,
                              const __grid_constant__ CUtensorMap tmDT, const AttnFp8Params p);
uint32_t attn_fp8_smem_bytes();

}  // namespace vc
