// common.cuh - workspace layout, launch bookkeeping and small numeric helpers
// shared by the kernels of libvcattn.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "vc_attn.h"

namespace vc {

constexpr int D = 128;      // head dimension
constexpr int TILE = 128;   // hardware block: rows of Q, keys of K/V, tokens of V-Smooth
constexpr int CHUNK32 = 32; // KV tiles whose block means are restored by one bf16 MMA

// Device status bits (workspace word).
constexpr uint32_t ST_TIMEOUT = 1u;

struct Shape {
  int B, H, N, BH, Nb, Npad, k, iters, R, Rpad, nch32;
  int km_nblk;   // k-means blocks per (b,h)
  int km_cpb;    // 128-token chunks per k-means block
  int kb_nchunk; // K-mean partial chunks per (b,h)
  unsigned flags;
};

// Byte offsets of the workspace arrays (all 256-byte aligned).
struct WsLayout {
  size_t gsync, perm, labels, cent, km_psum, km_pcnt, km_counter, kb_counter;
  size_t kbar_part, kbar;
  size_t q8, sq, k8, sk;
  size_t v8t, vscale, vexpo, vmean, amax_part, vq_counter, mut2, err;
  size_t rep_idx, rep_delta, deltat;
  size_t status;
  size_t cleared;  // bytes [0, cleared) hold the status word and counters: zeroed when a call starts
  size_t total;
};

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

Shape make_shape(int B, int H, int N, const vc_params &p, int repair_count);
WsLayout make_layout(const Shape &s);
WsLayout make_cluster_layout(const Shape &s);

// Bookkeeping: every launch in the library goes through this counter.
void count_launch();

// ---------------------------------------------------------------- numerics
__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }
__device__ __forceinline__ uint16_t f32_to_bf16_rn(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}
// Two floats -> two E4M3 codes (round to nearest even, saturating), lo in byte 0.
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  return static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}
// Exact value of two E4M3 codes (lo byte, hi byte).
__device__ __forceinline__ float2 e4m3x2_value(uint16_t codes) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(codes), __NV_E4M3);
  return __half22float2(*reinterpret_cast<__half2 *>(&h));
}
// Two floats -> two E2M1 (FP4) codes, round to nearest even, saturating to
// +/-6; lo in the low nibble.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp4x2(make_float2(lo, hi), __NV_E2M1, cudaRoundNearest));
}
// Exact value of two E2M1 codes (low nibble, high nibble).
__device__ __forceinline__ float2 e2m1x2_value(uint32_t codes) {
  __half2_raw h = __nv_cvt_fp4x2_to_halfraw2(static_cast<__nv_fp4x2_storage_t>(codes & 0xFFu), __NV_E2M1);
  return __half22float2(*reinterpret_cast<__half2 *>(&h));
}

// NVFP4 tile image of the values (one per 128-token tile of a head): the
// E4M3 block scales, 1024 bytes, byte 512*(jb/4) + 16*(c%32) + 4*(c/32) +
// jb%4 for channel c and 16-token block jb; then the E2M1 codes, 8192 bytes,
// channel rows of 64 bytes (token 2i in the low nibble of byte i) stored with
// the 64-byte swizzle: 8-row groups of 512 bytes, 16-byte chunk index XOR
// ((row / 2) mod 4).
constexpr int V4_SF_BYTES = 1024;
constexpr int V4_TILE_BYTES = V4_SF_BYTES + 128 * 64;
__host__ __device__ constexpr uint32_t sw64_off(int r, int ch) {
  return static_cast<uint32_t>((r >> 3) * 512 + (r & 7) * 64 + ((ch ^ ((r >> 1) & 3)) << 4));
}
__host__ __device__ constexpr uint32_t v4_sf_off(int c, int jb) {
  return static_cast<uint32_t>(512 * (jb >> 2) + 16 * (c & 31) + 4 * (c >> 5) + (jb & 3));
}

}  // namespace vc
