// attn_common.cuh - device helpers shared by the fused attention kernels
// (FP8 path and NVFP4-residual variant): elected issue, three-input max, frame
// rescale factors, the softmax warpgroups' named barriers and per-warp
// arrivals, the restore-chunk schedule and the O epilogue.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace vc {
namespace attn {

// One lane of a converged warp, chosen by elect.sync: the tcgen05 MMA groups
// are issued under this predicate so that the warp stays converged around them.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .b32 rx;\n\t.reg .pred px;\n\telect.sync rx|px, 0xffffffff;\n\t@px mov.s32 %0, 1;\n\t}"
      : "+r"(pred));
  return pred != 0;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Factor that moves a value from frame F_from to frame F_to >= F_from (both
// multiples of 8 byte units): the exact power of two 2^((F_from - F_to)/8).
__device__ __forceinline__ float frame_scale(float F_from, float F_to) {
  const int k = static_cast<int>((F_to - F_from) * 0.125f);
  return k > 126 ? 0.0f : __uint_as_float(static_cast<uint32_t>(127 - k) << 23);
}

__device__ __forceinline__ void softmax_bar256() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ void softmax_bar128(int g) { asm volatile("bar.sync %0, 128;" ::"r"(2 + g) : "memory"); }
// One arrive per warp on the barriers the softmax warpgroups signal (their
// expected count is 4 warps): the warp synchronizes first, which orders every
// lane's prior writes before lane 0's release.
__device__ __forceinline__ void warp_arrive(uint64_t *bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Restore chunks. Chunk X (KV tiles 32X .. 32X+31) is flushed by the tail of
// tile 32X+33, which reads l_{32X+31}; the chunks whose flush tile would lie
// past the last tile (one or two) are flushed after the loop.
__device__ __forceinline__ int first_epilogue_chunk(int T) { return T >= 34 ? (T - 34) / 32 + 1 : 0; }

// Epilogue of one softmax warp: its 32 rows of O_i (TMEM lanes of taddr,
// columns taddr .. taddr+127) become O = s_c * O_acc / l in bf16, one
// reciprocal of l per row. Each row thread stages its 256-byte row in `stg`
// (32 * 256 bytes of shared memory no longer read by anything; 16-byte chunk
// c of row r at chunk c XOR (r mod 16), so that neither the row-wise writes
// nor the chunk-wise reads conflict on banks); the warp then writes two whole
// rows per 16-byte store instruction. orow0: the O row of the warp's first
// row; rows >= nrows (past the head's last token) are not written.
__device__ __forceinline__ void store_o_rows(uint32_t taddr, const float *vscale, float l, uint8_t *stg,
                                             uint16_t *orow0, int nrows) {
  const int lane = threadIdx.x & 31;
  const float inv = __fdiv_rn(1.0f, l);
  uint8_t *mine = stg + lane * 256;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t v[32];
    tmem_ld32(taddr + 32 * i, v);
    tmem_wait_ld();
#pragma unroll
    for (int gg = 0; gg < 4; ++gg) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = 32 * i + 8 * gg + 2 * e;
        const float o0 = __uint_as_float(v[8 * gg + 2 * e]) * vscale[c] * inv;
        const float o1 = __uint_as_float(v[8 * gg + 2 * e + 1]) * vscale[c + 1] * inv;
        const __nv_bfloat162 ob = __floats2bfloat162_rn(o0, o1);
        w[e] = *reinterpret_cast<const uint32_t *>(&ob);
      }
      *reinterpret_cast<uint4 *>(mine + (((4 * i + gg) ^ (lane & 15)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  __syncwarp();
  const int ch = lane & 15;
#pragma unroll 4
  for (int it = 0; it < 16; ++it) {
    const int rr = 2 * it + (lane >> 4);
    if (rr < nrows)
      *reinterpret_cast<uint4 *>(orow0 + static_cast<size_t>(rr) * 128 + 8 * ch) =
          *reinterpret_cast<const uint4 *>(stg + rr * 256 + ((ch ^ (rr & 15)) << 4));
  }
}

}  // namespace attn
}  // namespace vc
