// attn_bf16.cuh - the in-library BF16 exact-softmax attention comparator.
#pragma once
#include <cstdint>
#include <cuda.h>

namespace vc {

struct AttnBf16Params {
  int N, Nb;
  float scale_log2;  // softmax_scale * log2(e)
  uint16_t *O;       // [BH][N][128] bf16
  uint32_t *status;  // device status word, or nullptr (no report)
};

__global__ void k_attn_ref_bf16(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                                const __grid_constant__ CUtensorMap tmV, const AttnBf16Params p);
uint32_t attn_bf16_smem_bytes();

}  // namespace vc
