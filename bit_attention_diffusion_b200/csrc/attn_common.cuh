// attn_common.cuh - device helpers shared by the fused attention kernels
// (FP8 path and NVFP4-residual variant): elected issue, three-input max, frame
// rescale factors, the softmax warpgroups' named barriers and per-warp
// arrivals, and the restore-chunk schedule.
#pragma once
#include <cstdint>

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

}  // namespace attn
}  // namespace vc
