// expcast.cuh - ExpCast-FP8 on the device (page "VC-Attention acelera atenção
// em modelos de vídeo de IA em até 3,58× sem retreinamento", section
// "ExpCast-FP8: eliminando o gargalo do softmax": an E4M3 byte is nearly a
// logarithm, so the probability byte is written from the log-domain score by
// one fused multiply-add instead of an exponential and a cast).
#pragma once
#include <cstdint>

namespace vc {

// 2^-24: scaling the fma by it puts the result on f16's subnormal grid.
constexpr float TWO_M24 = 5.9604644775390625e-08f;

// Two scores at once. y = fp32(acc * (alpha*2^-24) + (C - F)*2^-24) for both
// lanes (one packed f32x2 fma; the power-of-two scaling commutes with the
// rounding), then cvt.rn.relu.f16x2: y is a multiple of 2^-24 inside f16's
// subnormal range, so each f16 result's bit pattern is the integer
// RNE(fp32(acc*alpha + C - F)), clamped at 0 by relu - the E4M3 byte.
// Returns the two bytes in the low byte of each 16-bit half.
__device__ __forceinline__ uint32_t expcast2(float a0, float a1, float al0_24, float al1_24, float c24) {
  uint32_t h;
  asm("{\n\t.reg .b64 a, b, c, d;\n\t.reg .f32 y0, y1;\n\t"
      "mov.b64 a, {%1, %2};\n\tmov.b64 b, {%3, %4};\n\tmov.b64 c, {%5, %5};\n\t"
      "fma.rn.f32x2 d, a, b, c;\n\tmov.b64 {y0, y1}, d;\n\t"
      "cvt.rn.relu.f16x2.f32 %0, y1, y0;\n\t}"
      : "=r"(h)
      : "f"(a0), "f"(a1), "f"(al0_24), "f"(al1_24), "f"(c24));
  return h;
}

// Four scores sharing alpha -> four bytes packed little-endian.
__device__ __forceinline__ uint32_t expcast4(const float *a, float al24, float c24) {
  const uint32_t h01 = expcast2(a[0], a[1], al24, al24, c24);
  const uint32_t h23 = expcast2(a[2], a[3], al24, al24, c24);
  return __byte_perm(h01, h23, 0x6420);
}

}  // namespace vc
